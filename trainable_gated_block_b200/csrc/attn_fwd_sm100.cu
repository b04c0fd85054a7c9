// Gated block-sparse causal attention forward on the sm_100a tensor cores.
//
// SAS review (paper.oopus.info) §2.3, eq. o_SAS: o = softmax(q K_S^T + log g_S) V_S
// over the current block (gate 1, causal) and the kept history blocks (gate
// g_m = exp(s_m - LSE(s)), §2.4), computed tile by tile without the full
// logit matrix (§2.6). bf16 operands, fp32 accumulation, D = 128.
//
// Work item = (batch b, KV head h, query block i, head group tg): up to two
// 128-row Q tiles, each tile = 2 query heads x the 64 rows of block i. All
// query heads of a GQA group share the same kept blocks, so one K/V tile
// feeds both Q tiles. Persistent grid; items in order of decreasing cost.
//
// Warp roles (320 threads):
//   warp 0      TMA producer: Q tiles once per item, then K/V of two kept
//               blocks (128 keys) per step into a 2-stage ring, 128B-swizzled.
//   warp 1      TMEM owner and tcgen05 MMA issuer (one thread):
//               S_t = Q_t K^T into TMEM, then O_t += P_t V with P read from TMEM.
//   warps 2-5   softmax for Q tile 0, warps 6-9 for Q tile 1: each thread
//               owns one row (one TMEM lane); adds the block's log-gate to
//               the logits, masks the diagonal block causally, keeps an
//               online max/sum in the log2 domain, writes P (bf16) over S in
//               TMEM, rescales O in TMEM only when the max grows by > 2^8,
//               and finally writes o and the row LSE.
// TMEM (512 columns): S/P of tile t at [128t, 128t+128), O of tile t at
// [256+128t, 256+128t+128).
#include <cudaTypedefs.h>

#include "launch.h"
#include "sm100.cuh"

namespace sas {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kNS = 2;                              // K/V stages
constexpr int kThreads = 320;
constexpr uint32_t kBox = 64 * 128;                 // one TMA box: 64 rows x 128 B
constexpr uint32_t kQAtom = 2 * kBox;               // 128 rows x 128 B
constexpr uint32_t kQTile = 2 * kQAtom;             // 128 rows x 256 B
constexpr uint32_t kKVAtom = 2 * kBox;              // 128 keys x 128 B
constexpr uint32_t kKVTile = 2 * kKVAtom;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = 2 * kQTile;                          // 64 KB
constexpr uint32_t kOffV = kOffK + kNS * kKVTile;
constexpr uint32_t kOffBar = kOffV + kNS * kKVTile;             // 192 KB
constexpr uint32_t kSmemBytes = kOffBar + 1024 + 1024;          // + barriers + alignment slack
constexpr float kRescaleThreshold = 8.0f;           // log2 units: rescale O when the max grows by > 256x

struct Bars {
    uint64_t q_full, q_empty;
    uint64_t k_full[kNS], v_full[kNS], kv_empty[kNS];
    uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

struct Params {
    int B, S, Hq, Hkv, G, K, NQB, ntg, n_items;
    const int32_t* idx;
    const int32_t* cnt;
    const float* log_gate;
    float scale2;                       // sm_scale * log2(e)
    __nv_bfloat16* o;
    float* lse;
    int* status;
};

struct Item {
    int b, h, i, tg, nt, c, nb, ns;
    const int32_t* sel;
    const float* gate;
};

__device__ __forceinline__ Item item_of(const Params& p, int id) {
    Item it;
    const int per_i = p.B * p.Hkv * p.ntg;
    it.i = p.NQB - 1 - id / per_i;
    int r = id % per_i;
    it.tg = r % p.ntg;
    r /= p.ntg;
    it.h = r % p.Hkv;
    it.b = r / p.Hkv;
    it.nt = (4 * it.tg + 2 < p.G) ? 2 : 1;
    const long long row = ((long long)it.b * p.Hkv + it.h) * p.NQB + it.i;
    int c = p.cnt[row];
    const int cmax = min(p.K, it.i);
    c = max(0, min(c, cmax));
    it.c = c;
    it.nb = c + 1;
    it.ns = (it.nb + 1) >> 1;
    it.sel = p.idx + row * p.K;
    it.gate = p.log_gate + row * p.K;
    return it;
}

// Block k of the item's list (kept blocks ascending, then the current block).
// An out-of-range index is replaced by the current block, fully masked.
struct Blk {
    int j;
    bool valid, cur;
    float bias2;        // log-gate in log2 units
};
__device__ __forceinline__ Blk block_at(const Item& it, int k) {
    Blk r;
    if (k < it.c) {
        const int j = __ldg(it.sel + k);
        r.valid = (j >= 0 && j < it.i);
        r.j = r.valid ? j : it.i;
        r.cur = false;
        r.bias2 = r.valid ? __ldg(it.gate + k) * kLog2e : 0.f;
    } else {
        r.j = it.i;
        r.valid = true;
        r.cur = true;
        r.bias2 = 0.f;
    }
    return r;
}

__global__ void __launch_bounds__(kThreads, 1)
fwd_sm100_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &bars->abort;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_full[t], 128);
            mbar_init(&bars->o_full[t], 1);
            mbar_init(&bars->o_empty[t], 128);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&map_q);
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t sQ = smem_u32(smem + kOffQ);
    const uint32_t sK = smem_u32(smem + kOffK);
    const uint32_t sV = smem_u32(smem + kOffV);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kv_it = 0, q_it = 0;
            int last_stage_it[kNS] = {-1, -1};
            bool q_issued = false;
            for (int id = blockIdx.x; id < p.n_items && !*abort; id += gridDim.x) {
                const Item it = item_of(p, id);
                if (p.cnt[((long long)it.b * p.Hkv + it.h) * p.NQB + it.i] != it.c) flag_status(p.status, kStatusBadData);
                if (!mbar_wait(&bars->q_empty, (q_it & 1) ^ 1, abort, p.status)) break;
                mbar_expect_tx(&bars->q_full, (uint32_t)it.nt * 4 * kBox);
                for (int t = 0; t < it.nt; ++t)
                    for (int s = 0; s < 2; ++s) {
                        const int slot = 4 * it.tg + 2 * t + s;
                        const int hq = it.h * p.G + (slot < p.G ? slot : 0);
                        for (int a = 0; a < 2; ++a)
                            tma_load_3d(smem + kOffQ + t * kQTile + a * kQAtom + s * kBox, &map_q, &bars->q_full,
                                        a * 64, hq, it.b * p.S + it.i * 64);
                    }
                q_issued = true;
                ++q_it;
                for (int j = 0; j < it.ns; ++j, ++kv_it) {
                    const int st = kv_it % kNS;
                    if (!mbar_wait(&bars->kv_empty[st], ((kv_it / kNS) & 1) ^ 1, abort, p.status)) break;
                    const int nblk = (2 * j + 1 < it.nb) ? 2 : 1;
                    mbar_expect_tx(&bars->k_full[st], (uint32_t)nblk * 2 * kBox);
                    for (int bl = 0; bl < nblk; ++bl) {
                        const Blk bk = block_at(it, 2 * j + bl);
                        if (!bk.valid) flag_status(p.status, kStatusBadData);
                        for (int a = 0; a < 2; ++a)
                            tma_load_3d(smem + kOffK + st * kKVTile + a * kKVAtom + bl * kBox, &map_k,
                                        &bars->k_full[st], a * 64, it.h, it.b * p.S + bk.j * 64);
                    }
                    mbar_expect_tx(&bars->v_full[st], (uint32_t)nblk * 2 * kBox);
                    for (int bl = 0; bl < nblk; ++bl) {
                        const Blk bk = block_at(it, 2 * j + bl);
                        for (int a = 0; a < 2; ++a)
                            tma_load_3d(smem + kOffV + st * kKVTile + a * kKVAtom + bl * kBox, &map_v,
                                        &bars->v_full[st], a * 64, it.h, it.b * p.S + bk.j * 64);
                    }
                    last_stage_it[st] = (int)kv_it;
                }
            }
            if (*abort) {
                // let every copy this thread started land before the CTA exits
                for (int s = 0; s < kNS; ++s)
                    if (last_stage_it[s] >= 0) {
                        const uint32_t par = ((uint32_t)last_stage_it[s] / kNS) & 1;
                        volatile int no_abort = 0;
                        mbar_wait(&bars->k_full[s], par, &no_abort, nullptr);
                        mbar_wait(&bars->v_full[s], par, &no_abort, nullptr);
                    }
                if (q_issued) {
                    volatile int no_abort = 0;
                    mbar_wait(&bars->q_full, (q_it - 1) & 1, &no_abort, nullptr);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_pv = idesc_bf16(128, kD, false, true);
            uint32_t kv_it = 0, q_it = 0, p_it[2] = {0, 0}, oe_it[2] = {0, 0};
            auto issue_s = [&](int t, int st, int nk) {
                const uint32_t idesc = idesc_bf16(128, nk, false, false);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t a = sw128_desc(sQ + t * kQTile + (kk >> 2) * kQAtom + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = sw128_desc(sK + st * kKVTile + (kk >> 2) * kKVAtom + (kk & 3) * 32, 16, 1024);
                    mma_ss(tmem + t * 128, a, b, idesc, kk > 0);
                }
            };
            auto issue_pv = [&](int t, int st, int nk, bool acc) {
                for (int kk = 0; kk < nk / 16; ++kk) {
                    const uint64_t b = sw128_desc(sV + st * kKVTile + kk * 2048, kKVAtom, 1024);
                    mma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, b, idesc_pv, (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = true;
            for (int id = blockIdx.x; id < p.n_items && ok; id += gridDim.x) {
                const Item it = item_of(p, id);
                if (!(ok = mbar_wait(&bars->q_full, q_it & 1, abort, p.status))) break;
                ++q_it;
                tc_fence_after();
                {
                    const int st0 = kv_it % kNS;
                    if (!(ok = mbar_wait(&bars->k_full[st0], (kv_it / kNS) & 1, abort, p.status))) break;
                    tc_fence_after();
                    const int nk0 = (it.nb >= 2) ? 128 : 64;
                    for (int t = 0; t < it.nt; ++t) {
                        issue_s(t, st0, nk0);
                        mma_commit(&bars->s_full[t]);
                    }
                    if (it.ns == 1) mma_commit(&bars->q_empty);
                }
                for (int j = 0; j < it.ns && ok; ++j, ++kv_it) {
                    const int st = kv_it % kNS;
                    const int nk = (2 * j + 1 < it.nb) ? 128 : 64;
                    if (!(ok = mbar_wait(&bars->v_full[st], (kv_it / kNS) & 1, abort, p.status))) break;
                    tc_fence_after();
                    const bool more = j + 1 < it.ns;
                    const int st1 = (kv_it + 1) % kNS;
                    const int nk1 = (2 * (j + 1) + 1 < it.nb) ? 128 : 64;
                    for (int t = 0; t < it.nt && ok; ++t) {
                        if (!(ok = mbar_wait(&bars->p_full[t], p_it[t] & 1, abort, p.status))) break;
                        ++p_it[t];
                        if (j == 0) {
                            if (!(ok = mbar_wait(&bars->o_empty[t], (oe_it[t] & 1) ^ 1, abort, p.status))) break;
                            ++oe_it[t];
                        }
                        tc_fence_after();
                        issue_pv(t, st, nk, j > 0);
                        if (more) {
                            if (t == 0) {
                                if (!(ok = mbar_wait(&bars->k_full[st1], ((kv_it + 1) / kNS) & 1, abort, p.status)))
                                    break;
                                tc_fence_after();
                            }
                            issue_s(t, st1, nk1);
                            mma_commit(&bars->s_full[t]);
                        } else {
                            mma_commit(&bars->o_full[t]);
                        }
                    }
                    if (!ok) break;
                    if (j + 2 == it.ns) mma_commit(&bars->q_empty);
                    mma_commit(&bars->kv_empty[st]);
                }
            }
            // every MMA issued by this thread has finished before TMEM is freed
            mma_commit(&bars->drain);
            volatile int no_abort = 0;
            mbar_wait(&bars->drain, 0, &no_abort, nullptr);
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        const int t = (warp - 2) >> 2;                  // Q tile of this warpgroup
        const int quarter = warp & 3;                   // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;            // row of the Q tile = TMEM lane
        const int slot_in_tile = row >> 6, r_in = row & 63;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_base + t * 128;
        const uint32_t tO = tmem + lane_base + 256 + t * 128;
        uint32_t s_it = 0, o_it = 0;
        for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
            const Item it = item_of(p, id);
            if (t >= it.nt) continue;
            const int slot = 4 * it.tg + 2 * t + slot_in_tile;
            float m_ref = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < it.ns; ++j) {
                const Blk A = block_at(it, 2 * j);
                const bool hasB = 2 * j + 1 < it.nb;
                const Blk Bk = hasB ? block_at(it, 2 * j + 1) : A;
                if (!(ok = mbar_wait(&bars->s_full[t], s_it & 1, abort, p.status))) break;
                ++s_it;
                tc_fence_after();
                // pass 1: row max of the live logits, 32 columns at a time
                float mx = -INFINITY;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const Blk& bk = q < 2 ? A : Bk;
                    const bool blk_live = (q < 2 || hasB) && bk.valid;
                    uint32_t raw[32];
                    tmem_ld32(tS + q * 32, raw);
                    tmem_wait_ld();
                    if (!blk_live) continue;
                    float bm = -INFINITY;
                    if (bk.cur) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if ((q & 1) * 32 + e <= r_in) bm = fmaxf(bm, __uint_as_float(raw[e]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) bm = fmaxf(bm, __uint_as_float(raw[e]));
                    }
                    if (bm != -INFINITY) mx = fmaxf(mx, fmaf(bm, p.scale2, bk.bias2));
                }
                const float m_new = fmaxf(m_ref, mx);
                const bool need = m_new > m_ref + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need) && j > 0) {
                    const float f = need ? exp2f(m_ref - m_new) : 1.f;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t ov[32];
                        tmem_ld32(tO + q4 * 32, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
                        tmem_st32(tO + q4 * 32, ov);
                    }
                }
                if (need) {
                    l *= exp2f(m_ref - m_new);
                    m_ref = m_new;
                }
                const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
                // pass 2: P = exp2(logit - m) as bf16 pairs over the consumed S columns
                // (P columns [16q, 16q+16) lie inside S columns already read)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const Blk& bk = q < 2 ? A : Bk;
                    const bool blk_live = (q < 2 || hasB) && bk.valid;
                    uint32_t raw[32];
                    tmem_ld32(tS + q * 32, raw);
                    tmem_wait_ld();
                    uint32_t pk[16];
                    const float off = bk.bias2 - m_use;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int u0 = (q & 1) * 32 + 2 * e;
                        const bool live0 = blk_live && !(bk.cur && u0 > r_in);
                        const bool live1 = blk_live && !(bk.cur && u0 + 1 > r_in);
                        const float p0 = live0 ? exp2f(fmaf(__uint_as_float(raw[2 * e]), p.scale2, off)) : 0.f;
                        const float p1 = live1 ? exp2f(fmaf(__uint_as_float(raw[2 * e + 1]), p.scale2, off)) : 0.f;
                        l += p0 + p1;
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(tS + q * 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[t]);
            }
            if (!ok) break;
            if (!mbar_wait(&bars->o_full[t], o_it & 1, abort, p.status)) break;
            ++o_it;
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const bool store = slot < p.G;
            const int hq = it.h * p.G + slot;
            const long long orow = ((long long)it.b * p.S + (long long)it.i * 64 + r_in) * p.Hq + hq;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint32_t ov[32];
                tmem_ld32(tO + q4 * 32, ov);
                tmem_wait_ld();
                if (store) {
                    uint4* dst = reinterpret_cast<uint4*>(p.o + orow * kD + q4 * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv);
                        dst[v4] = w;
                    }
                }
            }
            if (store)
                p.lse[((long long)it.b * p.Hq + hq) * p.S + (long long)it.i * 64 + r_in] = (m_ref + log2f(l)) * kLn2;
            tc_fence_before();
            mbar_arrive(&bars->o_empty[t]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

}  // namespace

// [rows, H, D] bf16 viewed as 3-D (D, H, rows); 64 x 1 x 64 boxes, 128B swizzle.
bool make_head_map(CUtensorMap* map, const void* base, long long rows, int H, int D) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_fwd_sm100(const AttnArgs& a, void* o, float* lse, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    const long long rows = (long long)a.B * a.S;
    if (!make_head_map(&mq, a.q, rows, a.Hq, kD) || !make_head_map(&mk, a.k, rows, a.Hkv, kD) ||
        !make_head_map(&mv, a.v, rows, a.Hkv, kD))
        return cudaErrorInvalidValue;
    Params p;
    p.B = a.B;
    p.S = a.S;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.G = a.Hq / a.Hkv;
    p.K = a.K;
    p.NQB = a.S / 64;
    p.ntg = ((p.G + 1) / 2 + 1) / 2;
    p.n_items = a.B * a.Hkv * p.NQB * p.ntg;
    p.idx = a.idx;
    p.cnt = a.cnt;
    p.log_gate = a.log_gate;
    p.scale2 = a.sm_scale * kLog2e;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.status = a.status;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaFuncSetAttribute(fwd_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int grid = p.n_items < sms ? p.n_items : sms;
    fwd_sm100_kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, p);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace sas
