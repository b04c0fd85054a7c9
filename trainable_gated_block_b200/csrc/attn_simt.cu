// Gated block-sparse attention on the CUDA cores, fp32 arithmetic throughout.
//
// Forward: SAS review (paper.oopus.info) §2.3, eq. o_SAS - softmax over the
// logits sm_scale*q.k + log g, where log g is the kept block's log-gate and
// 0 on the current block (§2.4), with the causal mask on the current block;
// only kept blocks are visited, never the full matrix (§2.6).
// Backward: §2.6 - probabilities recomputed tile by tile from the saved row
// LSE; the gate gradient of a kept block is the sum of its logit gradients;
// ds follows from the Jacobian of s - LSE(s) (§2.4).
//
// This is the fp32 dtype path (tensor cores would round the operands). One
// CTA of 128 threads owns a 64-row stripe (b, hq, query block i): thread
// pairs split the head dimension of one query row. Key/value tiles of 64
// rows are staged in shared memory. Sequence b occupies token rows start_b ..
// start_b + len_b - 1; a partial last block is staged with zero rows past the
// end, its rows past the end are neither stored nor given gradient, and CTAs
// of blocks past the end return at once.
#include "common.cuh"
#include "launch.h"

namespace sas {
namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 16;              // keys per online-softmax update

// Loads a 64 x D tile (rows `row0..row0+63` of head h; rows from `nrows` on
// read as zero) into shared memory as fp32.
template <typename T, int D>
__device__ __forceinline__ void load_tile(float* dst, const T* src, long long row0, int H, int h, int nrows) {
    for (int e = threadIdx.x; e < kBlock * D; e += kThreads) {
        const int r = e / D, d = e % D;
        dst[r * (D + 1) + d] = r < nrows ? Elem<T>::load(src + ((row0 + r) * H + h) * (long long)D + d) : 0.f;
    }
}

// Tile list of query block i: kept history blocks (ascending), then block i.
__device__ __forceinline__ int tile_at(const int32_t* sel, int n_sel, int t, int i) {
    return t < n_sel ? sel[t] : i;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                int S, int Hq, int Hkv, int K, const int32_t* __restrict__ cu, long long Trows,
                const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
                const float* __restrict__ log_gate, float sm_scale,
                T* __restrict__ o, float* __restrict__ lse, int* status) {
    constexpr int HD = D / 2;
    extern __shared__ float smem[];
    float* Ks = smem;                               // [64][D+1]
    float* Vs = Ks + kBlock * (D + 1);              // [64][D+1]
    const int i = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
    const int NQB = (S + kBlock - 1) / kBlock, G = Hq / Hkv, h = hq / G;
    const int row = threadIdx.x >> 1, half = threadIdx.x & 1;
    const SeqRange sr = seq_range(cu, b, S, Trows, threadIdx.x == 0 ? status : nullptr);
    if (i * kBlock >= sr.len) return;               // block past the sequence's end
    const bool row_ok = i * kBlock + row < sr.len;
    const long long t = sr.start + (long long)i * kBlock + row;     // token row

    float qr[HD], acc[HD];
#pragma unroll
    for (int d = 0; d < HD; ++d) {
        qr[d] = row_ok ? Elem<T>::load(q + (t * Hq + hq) * D + half * HD + d) * sm_scale * kLog2e : 0.f;
        acc[d] = 0.f;
    }
    const long long sel_row = ((long long)(b * Hkv + h) * NQB + i);
    int n_sel = cnt[sel_row];
    if (n_sel < 0 || n_sel > min(K, i)) { flag_status(status, kStatusBadData); n_sel = max(0, min(n_sel, min(K, i))); }
    const int32_t* sel = idx + sel_row * K;
    const float* gates = log_gate + sel_row * K;

    float m = -INFINITY, l = 0.f;                   // running max / sum, log2 domain
    for (int tt = 0; tt <= n_sel; ++tt) {
        const int j = tile_at(sel, n_sel, tt, i);
        const bool cur = (tt == n_sel);
        const bool ok = cur || (j >= 0 && j < i);
        if (!ok) flag_status(status, kStatusBadData);
        __syncthreads();
        if (ok) {
            const int nr = min(kBlock, sr.len - j * kBlock);
            load_tile<T, D>(Ks, k, sr.start + (long long)j * kBlock, Hkv, h, nr);
            load_tile<T, D>(Vs, v, sr.start + (long long)j * kBlock, Hkv, h, nr);
        }
        __syncthreads();
        if (!ok) continue;
        const float bias = cur ? 0.f : gates[tt] * kLog2e;
        for (int u0 = 0; u0 < kBlock; u0 += kChunk) {
            float sc[kChunk];
            float cm = -INFINITY;
#pragma unroll
            for (int c = 0; c < kChunk; ++c) {
                const float* kr = Ks + (u0 + c) * (D + 1) + half * HD;
                float p = 0.f;
#pragma unroll
                for (int d = 0; d < HD; ++d) p = fmaf(qr[d], kr[d], p);
                p += __shfl_xor_sync(0xffffffffu, p, 1);
                sc[c] = (cur && (u0 + c) > row) ? -INFINITY : p + bias;
                cm = fmaxf(cm, sc[c]);
            }
            const float mn = fmaxf(m, cm);
            if (mn == -INFINITY) continue;
            const float scale = exp2f(m - mn);
            l *= scale;
#pragma unroll
            for (int d = 0; d < HD; ++d) acc[d] *= scale;
            m = mn;
#pragma unroll
            for (int c = 0; c < kChunk; ++c) {
                const float p = exp2f(sc[c] - m);
                l += p;
                const float* vr = Vs + (u0 + c) * (D + 1) + half * HD;
#pragma unroll
                for (int d = 0; d < HD; ++d) acc[d] = fmaf(p, vr[d], acc[d]);
            }
        }
    }
    if (!row_ok) return;
    const float inv = 1.f / l;
#pragma unroll
    for (int d = 0; d < HD; ++d) Elem<T>::store(o + (t * Hq + hq) * D + half * HD + d, acc[d] * inv);
    if (half == 0) lse[((long long)b * Hq + hq) * S + (long long)i * kBlock + row] = (m + log2f(l)) * kLn2;
}

// ---------------------------------------------------------------------------
// Backward.
// ---------------------------------------------------------------------------

struct BwdWs {
    float* Dr;      // [B, Hq, S]        rowsum(dO * O)
    float* gsum;    // [B, Hkv, NQB, K]  per kept block: sum of logit gradients
    float* dk;      // [B, S, Hkv, D]    fp32 accumulators
    float* dv;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline BwdWs carve(void* ws, int B, int S, long long T, int Hq, int Hkv, int D, int K) {
    char* p = static_cast<char*>(ws);
    BwdWs w;
    const int NQB = (S + kBlock - 1) / kBlock;
    w.Dr = reinterpret_cast<float*>(p); p += align256(sizeof(float) * (size_t)B * Hq * S);
    w.gsum = reinterpret_cast<float*>(p); p += align256(sizeof(float) * (size_t)B * Hkv * NQB * (size_t)(K > 0 ? K : 1));
    w.dk = reinterpret_cast<float*>(p); p += align256(sizeof(float) * (size_t)T * Hkv * D);
    w.dv = reinterpret_cast<float*>(p);
    return w;
}

template <typename T, int D>
__global__ void bwd_dot_kernel(const T* __restrict__ o, const T* __restrict__ dout, int B, int S, long long Trows,
                               int Hq, const int32_t* __restrict__ cu, float* __restrict__ Dr) {
    // One warp per (token, hq) row; Dr stored as [B, Hq, S] (rows of no sequence skipped).
    const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= Trows * Hq) return;
    const int hq = (int)(w % Hq);
    int b, t;
    if (!token_seq(cu, B, S, w / Hq, b, t)) return;
    float acc = 0.f;
    for (int d = lane; d < D; d += 32) acc = fmaf(Elem<T>::load(o + w * D + d), Elem<T>::load(dout + w * D + d), acc);
    acc = warp_sum(acc);
    if (lane == 0) Dr[((long long)b * Hq + hq) * S + t] = acc;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
bwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const T* __restrict__ dout, const float* __restrict__ lse,
                int S, int Hq, int Hkv, int K, const int32_t* __restrict__ cu, long long Trows,
                const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
                const float* __restrict__ log_gate, float sm_scale,
                T* __restrict__ dq, BwdWs ws, int* status) {
    constexpr int HD = D / 2;
    extern __shared__ float smem[];
    float* Ks = smem;                               // [64][D+1]
    float* Vs = Ks + kBlock * (D + 1);
    float* Qs = Vs + kBlock * (D + 1);              // this stripe's q rows
    float* dOs = Qs + kBlock * (D + 1);             // this stripe's dO rows
    float* Ps = dOs + kBlock * (D + 1);             // [64][65] probabilities
    float* dSs = Ps + kBlock * (kBlock + 1);        // [64][65] logit gradients
    float* red = dSs + kBlock * (kBlock + 1);       // [4] warp partial sums

    const int i = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
    const int NQB = (S + kBlock - 1) / kBlock, G = Hq / Hkv, h = hq / G;
    const int row = threadIdx.x >> 1, half = threadIdx.x & 1;
    const SeqRange sr = seq_range(cu, b, S, Trows, nullptr);
    if (i * kBlock >= sr.len) return;               // block past the sequence's end
    const int nrows = min(kBlock, sr.len - i * kBlock);
    const bool row_ok = row < nrows;
    const long long t = sr.start + (long long)i * kBlock + row;

    load_tile<T, D>(Qs, q, sr.start + (long long)i * kBlock, Hq, hq, nrows);
    load_tile<T, D>(dOs, dout, sr.start + (long long)i * kBlock, Hq, hq, nrows);
    __syncthreads();
    float qr[HD], dor[HD], dqa[HD];
#pragma unroll
    for (int d = 0; d < HD; ++d) {
        qr[d] = Qs[row * (D + 1) + half * HD + d] * sm_scale * kLog2e;
        dor[d] = dOs[row * (D + 1) + half * HD + d];
        dqa[d] = 0.f;
    }
    const float lse2 = row_ok ? lse[((long long)b * Hq + hq) * S + (long long)i * kBlock + row] * kLog2e : 0.f;
    const float Drow = row_ok ? ws.Dr[((long long)b * Hq + hq) * S + (long long)i * kBlock + row] : 0.f;

    const long long sel_row = ((long long)(b * Hkv + h) * NQB + i);
    int n_sel = cnt[sel_row];
    if (n_sel < 0 || n_sel > min(K, i)) { flag_status(status, kStatusBadData); n_sel = max(0, min(n_sel, min(K, i))); }
    const int32_t* sel = idx + sel_row * K;
    const float* gates = log_gate + sel_row * K;

    for (int tt = 0; tt <= n_sel; ++tt) {
        const int j = tile_at(sel, n_sel, tt, i);
        const bool cur = (tt == n_sel);
        const bool ok = cur || (j >= 0 && j < i);
        if (!ok) flag_status(status, kStatusBadData);
        __syncthreads();
        const int nk = min(kBlock, sr.len - j * kBlock);     // keys of block j inside the sequence
        if (ok) {
            load_tile<T, D>(Ks, k, sr.start + (long long)j * kBlock, Hkv, h, nk);
            load_tile<T, D>(Vs, v, sr.start + (long long)j * kBlock, Hkv, h, nk);
        }
        __syncthreads();
        if (!ok) continue;
        const float bias = cur ? 0.f : gates[tt] * kLog2e;
        float gpart = 0.f;
        for (int u = 0; u < kBlock; ++u) {
            const float* kr = Ks + u * (D + 1) + half * HD;
            const float* vr = Vs + u * (D + 1) + half * HD;
            float sdot = 0.f, pdot = 0.f;
#pragma unroll
            for (int d = 0; d < HD; ++d) { sdot = fmaf(qr[d], kr[d], sdot); pdot = fmaf(dor[d], vr[d], pdot); }
            sdot += __shfl_xor_sync(0xffffffffu, sdot, 1);
            pdot += __shfl_xor_sync(0xffffffffu, pdot, 1);
            const bool masked = (cur && u > row) || !row_ok;
            const float p = masked ? 0.f : exp2f(sdot + bias - lse2);
            const float dsv = p * (pdot - Drow);
#pragma unroll
            for (int d = 0; d < HD; ++d) dqa[d] = fmaf(dsv, kr[d], dqa[d]);
            if (half == 0) {
                Ps[row * (kBlock + 1) + u] = p;
                dSs[row * (kBlock + 1) + u] = dsv;
                gpart += dsv;
            }
        }
        __syncthreads();
        // Gate gradient of a kept block: sum of dS over the tile (and, via
        // atomics, over the query heads of the group).
        if (!cur) {
            float gw = warp_sum(gpart);
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = gw;
        }
        // dK_j += sm_scale * dS^T Q_i ; dV_j += P^T dO_i (thread: key row u, half of D).
        {
            constexpr int DC = 16;                      // head-dim columns per pass
            const int u = threadIdx.x >> 1;
            const long long krow = (sr.start + (long long)j * kBlock + u) * Hkv + h;
#pragma unroll 1
            for (int d0 = 0; d0 < HD; d0 += DC) {
                float dka[DC], dva[DC];
#pragma unroll
                for (int d = 0; d < DC; ++d) { dka[d] = 0.f; dva[d] = 0.f; }
                for (int r = 0; r < kBlock; ++r) {
                    const float pv = Ps[r * (kBlock + 1) + u];
                    const float dsv = dSs[r * (kBlock + 1) + u];
                    const float* qrow = Qs + r * (D + 1) + half * HD + d0;
                    const float* drow = dOs + r * (D + 1) + half * HD + d0;
#pragma unroll
                    for (int d = 0; d < DC; ++d) { dka[d] = fmaf(dsv, qrow[d], dka[d]); dva[d] = fmaf(pv, drow[d], dva[d]); }
                }
                if (u < nk) {                       // keys past the sequence's end: no store
#pragma unroll
                    for (int d = 0; d < DC; ++d) {
                        atomicAdd(ws.dk + krow * D + half * HD + d0 + d, dka[d] * sm_scale);
                        atomicAdd(ws.dv + krow * D + half * HD + d0 + d, dva[d]);
                    }
                }
            }
        }
        __syncthreads();
        if (!cur && threadIdx.x == 0)
            atomicAdd(ws.gsum + sel_row * K + tt, red[0] + red[1] + red[2] + red[3]);
    }
    if (!row_ok) return;
#pragma unroll
    for (int d = 0; d < HD; ++d) Elem<T>::store(dq + (t * Hq + hq) * D + half * HD + d, dqa[d] * sm_scale);
}

template <typename T>
__global__ void cast_kernel(const float* __restrict__ src, T* __restrict__ dst, long long n) {
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
        Elem<T>::store(dst + e, src[e]);
}

}  // namespace

// ds from the per-block gate gradients (shared by every backward path).
__global__ void ds_finalize_kernel(const float* __restrict__ s, int ld_s, const float* __restrict__ lse_s,
                                   const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
                                   const float* __restrict__ gsum, int rows, int NQB, int K, int Hkv,
                                   const int32_t* __restrict__ cu, int S, long long T, float* __restrict__ ds) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int i = (int)(row % NQB);
    if (i * kBlock >= seq_range(cu, (int)(row / NQB / Hkv), S, T, nullptr).len) {
        for (int j = lane; j < ld_s; j += 32) ds[row * (long long)ld_s + j] = 0.f;   // padding row
        return;
    }
    const int c = min(max(cnt[row], 0), min(K, i));
    float tot = 0.f;
    for (int m = lane; m < c; m += 32) tot += gsum[row * K + m];
    tot = warp_sum(tot);
    const float ls = lse_s[row];
    const float* srow = s + row * (long long)ld_s;
    float* drow = ds + row * (long long)ld_s;
    for (int j = lane; j < ld_s; j += 32)
        drow[j] = (j < i) ? -expf(srow[j] - ls) * tot : 0.f;
    __syncwarp();
    for (int m = lane; m < c; m += 32) {
        const int j = idx[row * K + m];
        if (j >= 0 && j < i) drow[j] += gsum[row * K + m];
    }
}

cudaError_t launch_ds_finalize(const float* s, int ld_s, const float* lse_s, const int32_t* idx,
                               const int32_t* cnt, const float* gsum, int B, int Hkv, int NQB, int K,
                               const int32_t* cu, int S, long long T, float* ds, cudaStream_t st) {
    const int rows = B * Hkv * NQB;
    ds_finalize_kernel<<<(rows + 7) / 8, 256, 0, st>>>(s, ld_s, lse_s, idx, cnt, gsum, rows, NQB, K, Hkv, cu, S, T,
                                                       ds);
    count_launches(1);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t fwd_go(const AttnArgs& a, void* o, float* lse, cudaStream_t st) {
    const size_t sm = sizeof(float) * 2 * kBlock * (D + 1);
    auto kern = fwd_simt_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    dim3 grid((a.S + kBlock - 1) / kBlock, a.Hq, a.B);
    kern<<<grid, kThreads, sm, st>>>((const T*)a.q, (const T*)a.k, (const T*)a.v, a.S, a.Hq, a.Hkv, a.K, a.cu, a.T,
                                     a.idx, a.cnt, a.log_gate, a.sm_scale, (T*)o, lse, a.status);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_fwd_simt(const AttnArgs& a, bool bf16, void* o, float* lse, cudaStream_t st) {
    if (bf16) return a.D == 64 ? fwd_go<__nv_bfloat16, 64>(a, o, lse, st) : fwd_go<__nv_bfloat16, 128>(a, o, lse, st);
    return a.D == 64 ? fwd_go<float, 64>(a, o, lse, st) : fwd_go<float, 128>(a, o, lse, st);
}

size_t bwd_simt_workspace(int B, int S, long long T, int Hq, int Hkv, int D, int K) {
    const int NQB = (S + kBlock - 1) / kBlock;
    return align256(sizeof(float) * (size_t)B * Hq * S) +
           align256(sizeof(float) * (size_t)B * Hkv * NQB * (size_t)(K > 0 ? K : 1)) +
           2 * align256(sizeof(float) * (size_t)T * Hkv * D);
}

template <typename T, int D>
static cudaError_t bwd_go(const BwdArgs& p, cudaStream_t st) {
    const AttnArgs& a = p.a;
    BwdWs ws = carve(p.workspace, a.B, a.S, a.T, a.Hq, a.Hkv, a.D, a.K);
    const int NQB = (a.S + kBlock - 1) / kBlock;
    cudaError_t e;
    e = cudaMemsetAsync(ws.gsum, 0, sizeof(float) * (size_t)a.B * a.Hkv * NQB * (size_t)(a.K > 0 ? a.K : 1), st);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(ws.dk, 0, sizeof(float) * (size_t)a.T * a.Hkv * D, st);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(ws.dv, 0, sizeof(float) * (size_t)a.T * a.Hkv * D, st);
    if (e != cudaSuccess) return e;
    const long long rows = a.T * a.Hq;
    bwd_dot_kernel<T, D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>((const T*)p.o, (const T*)p.dout, a.B, a.S, a.T,
                                                                     a.Hq, a.cu, ws.Dr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t sm = sizeof(float) * (4 * kBlock * (D + 1) + 2 * kBlock * (kBlock + 1) + 4);
    auto kern = bwd_simt_kernel<T, D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    dim3 grid(NQB, a.Hq, a.B);
    kern<<<grid, kThreads, sm, st>>>((const T*)a.q, (const T*)a.k, (const T*)a.v, (const T*)p.dout, p.lse,
                                     a.S, a.Hq, a.Hkv, a.K, a.cu, a.T, a.idx, a.cnt, a.log_gate, a.sm_scale,
                                     (T*)p.dq, ws, a.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long n = a.T * a.Hkv * D;
    cast_kernel<T><<<1184, 256, 0, st>>>(ws.dk, (T*)p.dk, n);
    cast_kernel<T><<<1184, 256, 0, st>>>(ws.dv, (T*)p.dv, n);
    count_launches(4);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_ds_finalize(p.s, p.ld_s, p.lse_s, a.idx, a.cnt, ws.gsum, a.B, a.Hkv, NQB, a.K, a.cu, a.S, a.T, p.ds,
                              st);
}

cudaError_t launch_bwd_simt(const BwdArgs& p, bool bf16, cudaStream_t st) {
    if (bf16) return p.a.D == 64 ? bwd_go<__nv_bfloat16, 64>(p, st) : bwd_go<__nv_bfloat16, 128>(p, st);
    return p.a.D == 64 ? bwd_go<float, 64>(p, st) : bwd_go<float, 128>(p, st);
}

}  // namespace sas
