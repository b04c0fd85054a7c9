// sas_decode_paged: one gated block-sparse decode step over a paged KV cache.
//
// SAS review (paper.oopus.info) §2.3, eq. o_SAS and §2.4: the query of
// sequence n (position kv_len-1) attends its current block c with gate 1 and
// its kept history blocks with their log-gates; §2.6: the KV cache lives in
// 64-token pages. Only the kept pages are read: each (page, KV head) is one
// contiguous 16 KiB tile of K and one of V.
//
// Split-KV: CTA (split, h, n) walks up to kBps of the (cnt + 1) blocks of
// (n, h) for all G query heads of the group, keeping an online softmax per
// head in the log2 domain, and writes an unnormalised partial (m, l, o).
// A combine kernel merges the splits. HBM-bound: every K/V byte is read once
// with 16-byte non-coherent loads; the math is fp32 FMA on the CUDA cores.
#include "common.cuh"
#include "launch.h"

namespace sas {
namespace {

constexpr int kThreads = 128;
constexpr int kBps = 4;                 // blocks per split
constexpr int kD = 128;
constexpr int kKStride = kD + 8;        // bf16 elements per padded K row (272 B)

inline int num_splits(int K) { return (K + 1 + kBps - 1) / kBps; }

struct Part {
    float* o;       // [N, Hq, splits, D]
    float* ml;      // [N, Hq, splits, 2]  (max, sum), log2 domain
};

inline Part carve(void* ws, int N, int Hq, int K) {
    Part p;
    const size_t no = (size_t)N * Hq * num_splits(K) * kD;
    p.o = static_cast<float*>(ws);
    p.ml = p.o + no;
    return p;
}

template <int G>
__global__ void __launch_bounds__(kThreads)
decode_split_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                    const __nv_bfloat16* __restrict__ vc, int num_pages,
                    const int32_t* __restrict__ page_table, int max_pages,
                    const int32_t* __restrict__ kv_len, int Hq, int Hkv, int K,
                    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
                    const float* __restrict__ log_gate, float sm_scale, Part part, int* status) {
    constexpr int ITEMS = (G * 64 + kThreads - 1) / kThreads;   // (head, dim-pair) items per thread
    __shared__ __align__(16) __nv_bfloat16 Ks[kBlock * kKStride];
    __shared__ __align__(16) __nv_bfloat16 Vs[kBlock * kD];
    __shared__ __align__(16) float Qs[G * kD];
    __shared__ float Ps[G * kBlock];
    __shared__ float m_s[G], l_s[G], scale_s[G];

    const int split = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int splits = gridDim.x;
    const int tid = threadIdx.x;
    const int L = kv_len[n];
    const bool len_ok = L >= 1 && L <= max_pages * kBlock;
    if (!len_ok) flag_status(status, kStatusBadData);
    const int c = len_ok ? (L - 1) / kBlock : 0;
    const long long sel_row = (long long)n * Hkv + h;
    int n_sel = cnt[sel_row];
    if (n_sel < 0 || n_sel > min(K, c)) { flag_status(status, kStatusBadData); n_sel = max(0, min(n_sel, min(K, c))); }
    const int t0 = split * kBps;
    const int t1 = len_ok ? min(t0 + kBps, n_sel + 1) : t0;

    for (int e = tid; e < G * kD; e += kThreads) {
        const int g = e / kD, d = e % kD;
        Qs[e] = __bfloat162float(q[((long long)n * Hq + h * G + g) * kD + d]) * sm_scale * kLog2e;
    }
    if (tid < G) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }
    float acc[ITEMS][2];
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) acc[it][0] = acc[it][1] = 0.f;

    for (int t = t0; t < t1; ++t) {
        const bool cur = (t == n_sel);
        const int j = cur ? c : idx[sel_row * K + t];
        int page = -1;
        if (j >= 0 && (cur || j < c) && j < max_pages) page = page_table[(long long)n * max_pages + j];
        const bool ok = page >= 0 && page < num_pages;
        if (!ok) flag_status(status, kStatusBadData);
        const int nvalid = cur ? L - c * kBlock : kBlock;
        const float bias = cur ? 0.f : log_gate[sel_row * K + t] * kLog2e;
        __syncthreads();                       // previous block fully consumed
        if (ok) {
            const uint4* ksrc = reinterpret_cast<const uint4*>(kc + ((long long)page * Hkv + h) * kBlock * kD);
            const uint4* vsrc = reinterpret_cast<const uint4*>(vc + ((long long)page * Hkv + h) * kBlock * kD);
            for (int e = tid; e < kBlock * kD / 8; e += kThreads) {
                const int r = e / (kD / 8), cc = e % (kD / 8);
                uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
                if (r < nvalid) { kv = __ldg(ksrc + e); vv = __ldg(vsrc + e); }
                *reinterpret_cast<uint4*>(Ks + r * kKStride + cc * 8) = kv;
                *reinterpret_cast<uint4*>(Vs + r * kD + cc * 8) = vv;
            }
        }
        __syncthreads();
        if (!ok) continue;
        // logits (log2 domain) for every (head, key) of the block
        for (int e = tid; e < G * kBlock; e += kThreads) {
            const int g = e / kBlock, u = e % kBlock;
            const uint4* kr = reinterpret_cast<const uint4*>(Ks + u * kKStride);
            const float4* qr = reinterpret_cast<const float4*>(Qs + g * kD);
            float dot = 0.f;
#pragma unroll
            for (int cc = 0; cc < kD / 8; ++cc) {
                const uint4 w = kr[cc];
                const float4 qa = qr[2 * cc], qb = qr[2 * cc + 1];
                float2 f;
                f = bf16x2_to_f32(w.x); dot = fmaf(qa.x, f.x, dot); dot = fmaf(qa.y, f.y, dot);
                f = bf16x2_to_f32(w.y); dot = fmaf(qa.z, f.x, dot); dot = fmaf(qa.w, f.y, dot);
                f = bf16x2_to_f32(w.z); dot = fmaf(qb.x, f.x, dot); dot = fmaf(qb.y, f.y, dot);
                f = bf16x2_to_f32(w.w); dot = fmaf(qb.z, f.x, dot); dot = fmaf(qb.w, f.y, dot);
            }
            Ps[e] = (u < nvalid) ? dot + bias : -INFINITY;
        }
        __syncthreads();
        // online softmax update, one warp per head
        for (int g = tid >> 5; g < G; g += kThreads / 32) {
            const int lane = tid & 31;
            const float a = Ps[g * kBlock + lane], b2 = Ps[g * kBlock + 32 + lane];
            const float bm = warp_max(fmaxf(a, b2));
            const float mo = m_s[g];
            const float mn = fmaxf(mo, bm);
            const float pa = exp2f(a - mn), pb = exp2f(b2 - mn);
            Ps[g * kBlock + lane] = pa;
            Ps[g * kBlock + 32 + lane] = pb;
            const float ps = warp_sum(pa + pb);
            if (lane == 0) {
                const float sc = exp2f(mo - mn);
                scale_s[g] = sc;
                l_s[g] = l_s[g] * sc + ps;
                m_s[g] = mn;
            }
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < ITEMS; ++it) {
            const int e = tid + it * kThreads;
            if (e < G * 64) {
                const int g = e / 64, dp = e % 64;
                const float sc = scale_s[g];
                float a0 = acc[it][0] * sc, a1 = acc[it][1] * sc;
                const float* pr = Ps + g * kBlock;
                const uint32_t* vcol = reinterpret_cast<const uint32_t*>(Vs) + dp;
#pragma unroll 8
                for (int u = 0; u < kBlock; ++u) {
                    const float p = pr[u];
                    const float2 f = bf16x2_to_f32(vcol[u * (kD / 2)]);
                    a0 = fmaf(p, f.x, a0);
                    a1 = fmaf(p, f.y, a1);
                }
                acc[it][0] = a0;
                acc[it][1] = a1;
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int e = tid + it * kThreads;
        if (e < G * 64) {
            const int g = e / 64, dp = e % 64;
            float* dst = part.o + (((long long)n * Hq + h * G + g) * splits + split) * kD + 2 * dp;
            dst[0] = acc[it][0];
            dst[1] = acc[it][1];
        }
    }
    if (tid < G) {
        float* ml = part.ml + (((long long)n * Hq + h * G + tid) * splits + split) * 2;
        ml[0] = m_s[tid];
        ml[1] = l_s[tid];
    }
}

__global__ void __launch_bounds__(kD)
decode_combine_kernel(Part part, int splits, int Hq, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
    const long long row = blockIdx.x;          // n * Hq + hq
    const int d = threadIdx.x;
    const float* ml = part.ml + row * splits * 2;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, ml[2 * s]);
    float Lsum = 0.f, acc = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float w = exp2f(ml[2 * s] - M);     // 0 for empty splits (m = -inf)
            Lsum = fmaf(ml[2 * s + 1], w, Lsum);
            acc = fmaf(part.o[(row * splits + s) * kD + d], w, acc);
        }
    }
    o[row * kD + d] = __float2bfloat16_rn(acc / Lsum);
    if (lse != nullptr && d == 0) lse[row] = (M + log2f(Lsum)) * kLn2;
}

template <int G>
cudaError_t go(const DecodeArgs& a, Part part, cudaStream_t st) {
    const int splits = num_splits(a.K);
    dim3 grid(splits, a.Hkv, a.N);
    decode_split_kernel<G><<<grid, kThreads, 0, st>>>(
        (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k_cache, (const __nv_bfloat16*)a.v_cache,
        a.num_pages, a.page_table, a.max_pages, a.kv_len, a.Hq, a.Hkv, a.K, a.idx, a.cnt,
        a.log_gate, a.sm_scale, part, a.status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<<<a.N * a.Hq, kD, 0, st>>>(part, splits, a.Hq, (__nv_bfloat16*)a.o, a.lse);
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace

size_t decode_workspace(int N, int Hq, int Hkv, int D, int K) {
    (void)Hkv; (void)D;
    const size_t per = (size_t)N * Hq * num_splits(K);
    return sizeof(float) * (per * kD + per * 2);
}

cudaError_t launch_decode(const DecodeArgs& a, void* workspace, cudaStream_t st) {
    Part part = carve(workspace, a.N, a.Hq, a.K);
    switch (a.Hq / a.Hkv) {
        case 1: return go<1>(a, part, st);
        case 2: return go<2>(a, part, st);
        case 4: return go<4>(a, part, st);
        case 5: return go<5>(a, part, st);
        case 8: return go<8>(a, part, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sas
