// Gated block-sparse causal attention backward on the sm_100a tensor cores.
//
// SAS review (paper.oopus.info) §2.6: the probabilities are recomputed tile
// by tile from the saved row LSE (never the full matrix), and the gradient
// of a kept block's gate is the sum of the logit gradients inside the block;
// §2.4, eq. log g: the scores receive it through the Jacobian of s - LSE(s)
// (ds_finalize_kernel). Per attended tile of query block i and key block j:
//   P = exp(sm_scale q.k + log g - lse),  dP = dO V^T,  dS = P (dP - Dr),
//   dQ += sm_scale dS K,  dK += sm_scale dS^T Q,  dV += P^T dO,
//   Gsum[i][slot(j)] += sum(dS)           (kept blocks only).
//
// Two tensor-core kernels, no floating-point atomics on dq/dk/dv:
//  * dq_kernel (query-stationary, like the forward): item = (b, h, i, head
//    pair), one 128-row Q tile (2 heads x 64 rows) whose Q and dO stay in
//    TMEM for the item. Per kept block: S = Q K^T and dP = dO V^T (A from
//    TMEM) into one of two TMEM buffers, dS to a swizzled shared-memory tile,
//    dQ += dS K accumulated in TMEM across the item. Also the per-block gate
//    gradients (warp sums of dS).
//  * dkv_kernel (key-stationary): item = (b, h, j); walks the query blocks
//    that attend block j (its own block and every block that kept it, from a
//    reverse index), one Q tile per step streamed through a 5-slot ring,
//    and accumulates dV^T = sum dO^T P and dK^T = sum Q^T dS in TMEM
//    (M = head dim); both softmax warpgroups work on every step.
// S and dP are computed twice (once per kernel) instead of once; in exchange
// nothing is reduced through global memory and dq/dk/dv are deterministic.
//
// Sequence b occupies token rows start_b .. start_b + len_b - 1 (a dense batch
// or a packed batch of different lengths); its last block may be partial.
// Query rows past the end get P = dS = 0 (they are read by the Q/dO boxes
// and dropped), key rows past the end get no dK/dV store, and items of blocks
// past the end are skipped by every role.
//
// Barrier discipline: every mbarrier phase is waited on in order by its
// consumer (a parity wait is exact only within one phase of the barrier), so
// "buffer is free again" barriers are waited on before every reuse of the
// buffer except the first.
#include "launch.h"
#include "sm100.cuh"

namespace sas {
namespace {

using namespace sm100;

constexpr int kD = 128;
// warp 0 TMA, warps 2-5 / 6-9 two softmax warpgroups, warps 1, 10, 11, 12
// four MMA-issuing warps (converged, elect.sync): one warp sustains about
// one tcgen05.mma per ~125 cycles whatever the tile width, so the MMAs of a
// step are spread over four warps that issue in parallel
constexpr int kThreads = 416;
__device__ __forceinline__ bool is_issuer_warp(int warp) { return warp == 1 || warp >= 10; }
// issuer slot 0..3 of an issuing warp: warps 1, 10, 11, 12
__device__ __forceinline__ int issuer_slot(int warp) { return warp == 1 ? 0 : warp - 9; }
constexpr uint32_t kBox = 64 * 128;        // TMA box: 64 rows x 128 B
constexpr uint32_t kTileAtom = 2 * kBox;   // 128 rows x 128 B (one 64-column half of a Q/dO tile)
constexpr uint32_t kTile = 2 * kTileAtom;  // 128 rows x 256 B
constexpr uint32_t kBlkAtom = kBox;        // 64 keys x 128 B
constexpr uint32_t kBlk = 2 * kBlkAtom;    // 64 keys x 256 B
constexpr uint32_t kRowTile = 128 * 128;   // 128 rows x 64 bf16 (P or dS of one Q tile)
constexpr uint32_t kHi = sm100::sdesc_hi(1024);   // high descriptor word: 8-row groups 1024 B apart

// ------------------------------------------------------------------ shared
struct Params {
    int B, S, Hq, Hkv, G, K, NQB, n_items, ntile;
    const int32_t* cu;      // packed sequence bounds [B + 1], or nullptr (dense)
    long long T;            // token rows of q/k/v/dO
    const int32_t* idx;
    const int32_t* cnt;
    const float* log_gate;
    const float* lse;       // [B, Hq, S]
    const float* Dr;        // [B, Hq, S]
    const int32_t* rlist;   // [B, Hkv, NQB, NQB]: (i << 16) | slot, slot 0xFFFF = own block
    const int32_t* rcount;  // [B, Hkv, NQB]
    const int32_t* order;   // dk/dv items sorted by decreasing step count
    float scale2;           // sm_scale * log2(e)
    float sm_scale;
    float inv_scale;        // 1 / sm_scale
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* gsum;            // [B, Hkv, NQB, K]
    int* status;
};

// Elementwise part of the backward for the 32 keys [32 hf, 32 hf + 32) of
// one query row, from its S (sv) and dP (pv) values read out of TMEM:
//   P = 2^(S * sm_scale * log2 e + off),  dS' = P * (dP * sm_scale - Dr * sm_scale)
// where off = log2 g - lse (log2 units) or -inf for a dead row; keys above
// `lim` are masked (the diagonal block, kMask). dS' (dS times sm_scale) is
// rounded to bf16 into the row's 128-byte-swizzled tile, and P too when a P
// tile is given (the dq kernel gives none). Returns the row's sum of dS'.
template <bool kMask>
__device__ __forceinline__ float pds_half(const uint32_t (&sv)[32], const uint32_t (&pv)[32], int hf, float scale2,
                                          float off, float sm_scale, float drs, int lim, uint8_t* bufP,
                                          uint8_t* bufS, int row) {
    // two keys per f32x2 instruction (same rounding per key as the scalar forms)
    const unsigned long long sc2 = f2_pack(scale2, scale2), off2 = f2_pack(off, off);
    const unsigned long long sm2 = f2_pack(sm_scale, sm_scale), nd2 = f2_pack(-drs, -drs);
    unsigned long long gs2[2] = {0ull, 0ull};       // 2 independent chains of pairs
#pragma unroll
    for (int c = 0; c < 4; ++c) {                 // 16-byte chunk = keys 8c .. 8c+7 of the half
        uint32_t pp[4], dd[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
            const int e = 8 * c + 2 * e2;
            float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, off2));
            if (kMask) {
                x.x = (32 * hf + e > lim) ? -INFINITY : x.x;
                x.y = (32 * hf + e + 1 > lim) ? -INFINITY : x.y;
            }
            const float p0 = fast_exp2(x.x), p1 = fast_exp2(x.y);
            const unsigned long long dp = f2_fma(f2_pack(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1])), sm2, nd2);
            const unsigned long long ds = f2_mul(f2_pack(p0, p1), dp);
            gs2[e2 & 1] = f2_add(gs2[e2 & 1], ds);
            const float2 d = f2_unpack(ds);
            pp[e2] = pack_bf16x2(p0, p1);
            dd[e2] = pack_bf16x2(d.x, d.y);
        }
        const int ch = 4 * hf + c;
        if (bufP) *reinterpret_cast<uint4*>(bufP + sw128_offset(row, ch)) = make_uint4(pp[0], pp[1], pp[2], pp[3]);
        *reinterpret_cast<uint4*>(bufS + sw128_offset(row, ch)) = make_uint4(dd[0], dd[1], dd[2], dd[3]);
    }
    const float2 g = f2_unpack(f2_add(gs2[0], gs2[1]));
    return g.x + g.y;
}

// ===================================================================== dq
namespace dqk {

// One 128-row Q tile (two heads x 64 rows of query block i) per item; Q and
// dO stay in TMEM for the whole item (A operands of S = Q K^T, dP = dO V^T),
// the kept K/V blocks stream through a 4-stage ring.
constexpr int kNS = 4;
constexpr uint32_t kStage = 2 * kBlk;                      // K block, V block
constexpr uint32_t kOffKV = 0;
constexpr uint32_t kOffQs = kOffKV + kNS * kStage;         // staging: Q tile, dO tile (TMA -> TMEM)
constexpr uint32_t kOffDS = kOffQs + 2 * kTile;            // 2 dS tiles (one per warpgroup)
constexpr uint32_t kOffBar = kOffDS + 2 * kRowTile;        // 224 KB
constexpr uint32_t kSmem = kOffBar + 1024 + 1024;
// TMEM columns
constexpr uint32_t kTmQ = 0, kTmO = 64, kTmS = 128, kTmDQ = 384;   // S/dP buffer u at kTmS + 128 u (S, dP + 64)

// warps: 0 TMA; 2-5 / 6-9 softmax warpgroups 0 / 1 (warpgroup u takes the
// blocks of odd / even position in the CTA's block stream); issuing warps
// 1, 10: S of stream parity 0 / 1; 11, 12: dP of parity 0 / 1; 13: dQ
constexpr int kThreadsDq = 448;

struct Bars {
    uint64_t qs_full, qs_empty, qt_full, qt_free;       // Q/dO staging full/empty, TMEM copy full/free
    uint64_t k_full[kNS], v_full[kNS], kv_empty[kNS];
    uint64_t s_full[2], tm_free[2], ds_full[2], ds_empty[2];
    uint64_t dq_full, dq_empty;
    uint64_t drain[5];
    uint32_t tmem_base;
    int abort;
};

struct Item {
    int b, h, i, t, c, nb, len;
    long long row;     // selection row (b, h, i)
    long long start;   // first token row of the sequence
    bool skip;         // query block past the sequence's end
};

__device__ __forceinline__ Item item_of(const Params& p, int id) {
    Item it;
    // head by head (the CTAs working at the same time share one head's K/V in
    // L2), query blocks from the last (longest items) down, then the tile
    const int per_bh = p.NQB * p.ntile;
    const int bh = id / per_bh, r = id % per_bh;
    it.i = p.NQB - 1 - r / p.ntile;
    it.t = r % p.ntile;
    it.h = bh % p.Hkv;
    it.b = bh / p.Hkv;
    it.row = ((long long)it.b * p.Hkv + it.h) * p.NQB + it.i;
    const SeqRange sr = seq_range(p.cu, it.b, p.S, p.T, nullptr);
    it.start = sr.start;
    it.len = sr.len;
    it.skip = it.i * 64 >= it.len;
    it.c = it.skip ? 0 : max(0, min(p.cnt[it.row], min(p.K, it.i)));
    it.nb = it.c + 1;
    return it;
}

// This CTA's next item at or after `id` (stride gridDim.x) that is not past
// its sequence's end; every role walks the same list.
__device__ __forceinline__ int live_item(const Params& p, int id) {
    while (id < p.n_items && item_of(p, id).skip) id += gridDim.x;
    return id;
}

struct Blk {
    int j;
    bool valid, cur;
    float bias2;
};
__device__ __forceinline__ Blk block_at(const Params& p, const Item& it, int k) {
    Blk r;
    if (k < it.c) {
        const int j = __ldg(p.idx + it.row * p.K + k);
        const float lg = __ldg(p.log_gate + it.row * p.K + k);   // issued without waiting for j
        r.valid = (j >= 0 && j < it.i);
        r.j = r.valid ? j : it.i;
        r.cur = false;
        r.bias2 = r.valid ? lg * kLog2e : 0.f;
    } else {
        r.j = it.i;
        r.valid = true;
        r.cur = true;
        r.bias2 = 0.f;
    }
    return r;
}

__global__ void __launch_bounds__(kThreadsDq, 1)
dq_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
          const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &bars->abort;
    if (threadIdx.x == 0) {
        mbar_init(&bars->qs_full, 1);
        mbar_init(&bars->qs_empty, 256);                 // both warpgroups copied their half
        mbar_init(&bars->qt_full, 256);
        mbar_init(&bars->qt_free, 4);                    // the four S / dP warps
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->kv_empty[s], 3);            // S, dP and dQ warps
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(&bars->s_full[u], 2);              // S and dP warps
            mbar_init(&bars->tm_free[u], 128);
            mbar_init(&bars->ds_full[u], 128);
            mbar_init(&bars->ds_empty[u], 1);
        }
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 256);
        for (int w = 0; w < 5; ++w) mbar_init(&bars->drain[w], 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t s_base = smem_u32(smem);

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0) {
            uint32_t kb = 0, qn = 0;
            int last_kv[kNS] = {-1, -1, -1, -1};
            bool q_pending = false;
            // Q/dO tile of item `id` into the staging buffer (once the previous one
            // has been copied to TMEM)
            auto load_qd = [&](int id) -> bool {
                const Item it = item_of(p, id);
                if (!mbar_wait(&bars->qs_empty, (qn & 1) ^ 1, abort, p.status)) return false;
                mbar_expect_tx(&bars->qs_full, 8 * kBox);
                for (int s = 0; s < 2; ++s) {
                    const int slot = 2 * it.t + s;
                    const int hq = it.h * p.G + (slot < p.G ? slot : 0);
                    for (int a = 0; a < 2; ++a) {
                        const uint32_t off = a * kTileAtom + s * kBox;
                        tma_load_3d(smem + kOffQs + off, &map_q, &bars->qs_full, a * 64, hq, (int)(it.start + it.i * 64));
                        tma_load_3d(smem + kOffQs + kTile + off, &map_do, &bars->qs_full, a * 64, hq,
                                    (int)(it.start + it.i * 64));
                    }
                }
                ++qn;
                q_pending = true;
                return true;
            };
            if (p.cu != nullptr)           // check the packed bounds once (flags a bad sequence)
                for (int bb = 0; bb < p.B; ++bb) seq_range(p.cu, bb, p.S, p.T, p.status);
            const int first = live_item(p, blockIdx.x);
            bool ok = first >= p.n_items || load_qd(first);
            for (int id = first; id < p.n_items && ok && !*abort; id = live_item(p, id + gridDim.x)) {
                const Item it = item_of(p, id);
                const int nxt = live_item(p, id + gridDim.x);
                const int k_next = min(1, it.nb - 1);   // the next item's Q/dO goes out after this block
                for (int k = 0; k < it.nb && ok; ++k, ++kb) {
                    const int st = kb % kNS;
                    if (!(ok = mbar_wait(&bars->kv_empty[st], ((kb / kNS) & 1) ^ 1, abort, p.status))) break;
                    const Blk bk = block_at(p, it, k);
                    if (!bk.valid) flag_status(p.status, kStatusBadData);
                    mbar_expect_tx(&bars->k_full[st], 2 * kBox);
                    for (int a = 0; a < 2; ++a)
                        tma_load_3d(smem + kOffKV + st * kStage + a * kBlkAtom, &map_k, &bars->k_full[st], a * 64, it.h,
                                    (int)(it.start + bk.j * 64));
                    mbar_expect_tx(&bars->v_full[st], 2 * kBox);
                    for (int a = 0; a < 2; ++a)
                        tma_load_3d(smem + kOffKV + st * kStage + kBlk + a * kBlkAtom, &map_v, &bars->v_full[st],
                                    a * 64, it.h, (int)(it.start + bk.j * 64));
                    last_kv[st] = (int)kb;
                    if (k == k_next && nxt < p.n_items) ok = load_qd(nxt);
                }
            }
            if (*abort) {           // let every copy in flight land before the CTA exits
                volatile int no_abort = 0;
                for (int s = 0; s < kNS; ++s)
                    if (last_kv[s] >= 0) {
                        const uint32_t par = ((uint32_t)last_kv[s] / kNS) & 1;
                        mbar_wait(&bars->k_full[s], par, &no_abort, nullptr);
                        mbar_wait(&bars->v_full[s], par, &no_abort, nullptr);
                    }
                if (q_pending) mbar_wait(&bars->qs_full, (qn - 1) & 1, &no_abort, nullptr);
            }
        }
    } else if (warp == 1 || warp >= 10) {
        // ----------------------------------------------------- issuing warps
        const int slot = warp == 1 ? 0 : warp - 9;      // 0, 1: S parity 0/1; 2, 3: dP parity 0/1; 4: dQ
        uint32_t kb = 0, qn = 0;
        bool ok = true;
        if (slot < 4) {
            const int u = slot & 1;
            const bool is_s = slot < 2;
            const uint32_t id_s = idesc_bf16(128, 64, false, false);
            const uint32_t a_tm = tmem + (is_s ? kTmQ : kTmO);
            const uint32_t d_tm = tmem + kTmS + 128 * u + (is_s ? 0u : 64u);
            const uint32_t b_off = is_s ? 0u : kBlk;
            uint32_t n_mine = 0;
            for (int id = live_item(p, blockIdx.x); id < p.n_items && ok; id = live_item(p, id + gridDim.x), ++qn) {
                const Item it = item_of(p, id);
                // this item's Q and dO are in TMEM
                if (!(ok = mbar_wait_warp(&bars->qt_full, qn & 1, abort, p.status))) break;
                tc_fence_after();
                for (int k = 0; k < it.nb && ok; ++k, ++kb) {
                    if ((kb & 1) != (uint32_t)u) continue;
                    const int st = kb % kNS;
                    uint64_t* fb = is_s ? &bars->k_full[st] : &bars->v_full[st];
                    if (!(ok = mbar_wait_warp(fb, (kb / kNS) & 1, abort, p.status))) break;
                    // warpgroup u has read its previous S / dP out of TMEM
                    if (n_mine > 0 && !(ok = mbar_wait_warp(&bars->tm_free[u], (n_mine - 1) & 1, abort, p.status)))
                        break;
                    ++n_mine;
                    tc_fence_after();
                    const uint32_t b_lo = sdesc_lo(s_base + kOffKV + st * kStage + b_off, 16);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t bo = (kk >> 2) * kBlkAtom + (kk & 3) * 32;
                        mma_ts_e(d_tm, a_tm + kk * 8, b_lo + (bo >> 4), kHi, id_s, kk > 0);
                    }
                    mma_commit_e(&bars->s_full[u]);
                    mma_commit_e(&bars->kv_empty[st]);
                }
                if (!ok) break;
                mma_commit_e(&bars->qt_free);           // done reading this item's Q / dO in TMEM
            }
        } else {
            // dQ += dS K (SS: A = dS tile of the block's warpgroup, B = K MN-major)
            const uint32_t id_dq = idesc_bf16(128, kD, false, true);
            uint32_t ds_n[2] = {0, 0};
            for (int id = live_item(p, blockIdx.x); id < p.n_items && ok; id = live_item(p, id + gridDim.x), ++qn) {
                const Item it = item_of(p, id);
                for (int k = 0; k < it.nb && ok; ++k, ++kb) {
                    const int u = kb & 1, st = kb % kNS;
                    if (!(ok = mbar_wait_warp(&bars->ds_full[u], ds_n[u] & 1, abort, p.status))) break;
                    ++ds_n[u];
                    // the previous item's dQ has been read out of TMEM
                    if (k == 0 && !(ok = mbar_wait_warp(&bars->dq_empty, (qn & 1) ^ 1, abort, p.status))) break;
                    tc_fence_after();
                    const uint32_t ds_lo = sdesc_lo(s_base + kOffDS + u * kRowTile, 16);     // K-major dS
                    const uint32_t kt_lo = sdesc_lo(s_base + kOffKV + st * kStage, kBlkAtom); // MN-major K
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss_e(tmem + kTmDQ, ds_lo + ((kk * 32) >> 4), kHi, kt_lo + ((kk * 2048) >> 4), kHi, id_dq,
                                 (k > 0 || kk > 0) ? 1u : 0u);
                    mma_commit_e(&bars->ds_empty[u]);
                    mma_commit_e(&bars->kv_empty[st]);
                    if (k + 1 == it.nb) mma_commit_e(&bars->dq_full);
                }
            }
        }
        mma_commit_e(&bars->drain[slot]);
        volatile int no_abort = 0;
        mbar_wait(&bars->drain[slot], 0, &no_abort, nullptr);
    } else {
        // ------------------------------------------------ softmax warpgroups
        const int u = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int slot_in_tile = row >> 6, r_in = row & 63;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_base + kTmS + 128 * u;
        const uint32_t tP = tS + 64;
        uint8_t* ds_tile = smem + kOffDS + u * kRowTile;
        uint32_t kb = 0, qn = 0, s_it = 0, ds_n = 0;
        bool ok = true;
        // copy this warpgroup's half of staged tile number n (0: Q, 1: dO) into TMEM
        // once the S / dP warps are done with the previous item's
        auto copy_qd = [&](uint32_t n) -> bool {
            if (n > 0 && !mbar_wait(&bars->qt_free, (n - 1) & 1, abort, p.status)) return false;
            if (!mbar_wait(&bars->qs_full, n & 1, abort, p.status)) return false;
            const uint8_t* src = smem + kOffQs + u * kTile;
            const uint32_t dst = tmem + lane_base + (u == 0 ? kTmQ : kTmO);
#pragma unroll
            for (int a = 0; a < 2; ++a) {               // dims [64 a, 64 a + 64) -> 32 packed columns
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 w = *reinterpret_cast<const uint4*>(src + a * kTileAtom + sw128_offset(row, c));
                    v[4 * c] = w.x;
                    v[4 * c + 1] = w.y;
                    v[4 * c + 2] = w.z;
                    v[4 * c + 3] = w.w;
                }
                tmem_st32(dst + 32 * a, v);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->qs_empty);
            mbar_arrive(&bars->qt_full);
            return true;
        };
        if (live_item(p, blockIdx.x) < p.n_items) ok = copy_qd(0);
        for (int id = live_item(p, blockIdx.x); id < p.n_items && ok; id = live_item(p, id + gridDim.x), ++qn) {
            const Item it = item_of(p, id);
            const int slot = 2 * it.t + slot_in_tile;
            // rows of an absent head, or past the sequence's end, contribute nothing
            const bool row_ok = slot < p.G && it.i * 64 + r_in < it.len;
            const int hq = it.h * p.G + (slot < p.G ? slot : 0);
            const long long lrow = ((long long)it.b * p.Hq + hq) * p.S + (long long)it.i * 64 + r_in;
            const float lse2 = row_ok ? p.lse[lrow] * kLog2e : 0.f;
            const float drs = row_ok ? p.Dr[lrow] * p.sm_scale : 0.f;
            // this warpgroup's blocks: stream positions kb + k with (kb + k) % 2 == u
            int k = (int)((u - (int)(kb & 1)) & 1);
            Blk nxt;
            if (k < it.nb) nxt = block_at(p, it, k);
            for (; k < it.nb; k += 2) {
                const Blk bk = nxt;
                if (k + 2 < it.nb) nxt = block_at(p, it, k + 2);
                if (!(ok = mbar_wait(&bars->s_full[u], s_it & 1, abort, p.status))) break;
                ++s_it;
                tc_fence_after();
                // log2 domain; rows of an absent head (or a bad block) get -inf: P = dS = 0
                const float off = (row_ok && bk.valid) ? bk.bias2 - lse2 : -INFINITY;
                float gs = 0.f;                           // sum of dS * sm_scale over the row's keys
                // dQ of this warpgroup's previous block has finished reading the dS tile
                if (ds_n > 0 && !(ok = mbar_wait(&bars->ds_empty[u], (ds_n - 1) & 1, abort, p.status))) break;
                ++ds_n;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {          // keys [32 hf, 32 hf + 32)
                    uint32_t sv[32], pv[32];
                    tmem_ld32(tS + 32 * hf, sv);
                    tmem_ld32(tP + 32 * hf, pv);
                    tmem_wait_ld();
                    if (hf == 1) {
                        tc_fence_before();
                        mbar_arrive(&bars->tm_free[u]);   // S/dP columns may be refilled
                    }
                    if (bk.cur)                           // causal mask on the diagonal block
                        gs += pds_half<true>(sv, pv, hf, p.scale2, off, p.sm_scale, drs, r_in, nullptr, ds_tile, row);
                    else
                        gs += pds_half<false>(sv, pv, hf, p.scale2, off, p.sm_scale, drs, 63, nullptr, ds_tile, row);
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars->ds_full[u]);
                if (!bk.cur && bk.valid) {
                    gs = warp_sum(gs);
                    if (lane == 0) atomicAdd(p.gsum + it.row * p.K + k, gs * p.inv_scale);
                }
            }
            if (!ok) break;
            kb += it.nb;
            // the next item's Q / dO go into TMEM first, so that its S / dP start
            // while this item's dQ is written out
            if (live_item(p, id + gridDim.x) < p.n_items && !(ok = copy_qd(qn + 1))) break;
            // dQ of the item: warpgroup u writes dims [64 u, 64 u + 64) of its rows
            if (!(ok = mbar_wait(&bars->dq_full, qn & 1, abort, p.status))) break;
            tc_fence_after();
            const long long orow = (it.start + (long long)it.i * 64 + r_in) * p.Hq + hq;
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                uint32_t ov[32];
                tmem_ld32(tmem + lane_base + kTmDQ + 64 * u + 32 * q2, ov);
                tmem_wait_ld();
                if (row_ok) {
                    uint4* dst = reinterpret_cast<uint4*>(p.dq + orow * kD + 64 * u + 32 * q2);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]), __uint_as_float(ov[8 * v4 + 1]));
                        w.y = pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]), __uint_as_float(ov[8 * v4 + 3]));
                        w.z = pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]), __uint_as_float(ov[8 * v4 + 5]));
                        w.w = pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]), __uint_as_float(ov[8 * v4 + 7]));
                        dst[v4] = w;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->dq_empty);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace dqk

// ==================================================================== dk, dv
namespace dkv {

// K_j, V_j stay in shared memory for the item; the steps' Q and dO tiles
// (32 KiB each) stream through a ring of five slots, Q of step g in slot
// 2g mod 5 and dO in slot 2g+1 mod 5, so two and a half steps are in flight.
constexpr uint32_t kOffK = 0;                      // K_j: 64 keys x 256 B
constexpr uint32_t kOffV = kBlk;                   // V_j
constexpr uint32_t kOffRing = 2 * kBlk;
constexpr int kSlots = 5;
constexpr uint32_t kOffP = kOffRing + kSlots * kTile;    // P tile, then dS tile of the current step
constexpr uint32_t kOffDS = kOffP + kRowTile;
constexpr uint32_t kOffBar = kOffDS + kRowTile;          // 224 KB
constexpr uint32_t kSmem = kOffBar + 1024 + 1024;
// TMEM columns: S/dP buffer b (steps of parity b) at 128 b (S, dP + 64); dV^T, dK^T accumulators
constexpr uint32_t kTmAccV = 256, kTmAccK = 320;

// warps: 0 TMA; 2-5 / 6-9 softmax warpgroups 0 / 1 (both on every step, keys
// [32 w, 32 w + 32); each writes P, then dS); issuing warps 1: S = Q K^T,
// 10: dP = dO V^T, 11: dV^T += dO^T P (as soon as P is written, so the dO
// slot is released while dS is computed), 12: dK^T += Q^T dS

struct Bars {
    uint64_t kv_full, kv_empty;
    uint64_t q_full[kSlots], o_full[kSlots], slot_empty[kSlots];
    uint64_t s_full[2], tm_free[2], pds_full, pds_empty, p_full, p_empty;
    uint64_t acc_full, acc_empty;
    uint64_t drain[4];
    uint32_t tmem_base;
    int abort;
};

// Item (b, h, j) and its sequence's token range; len = 0 marks an item whose
// key block lies past the sequence's end (skipped by every role).
struct KItem {
    int b, h, j, len;
    long long bh, start;
};
__device__ __forceinline__ KItem item_of(const Params& p, int id) {
    KItem it;
    it.j = id % p.NQB;
    const int r = id / p.NQB;
    it.h = r % p.Hkv;
    it.b = r / p.Hkv;
    it.bh = (long long)it.b * p.Hkv + it.h;
    const SeqRange sr = seq_range(p.cu, it.b, p.S, p.T, nullptr);
    it.start = sr.start;
    it.len = it.j * 64 < sr.len ? sr.len : 0;
    return it;
}

__device__ __forceinline__ int n_entries(const Params& p, const KItem& it) {
    if (it.len == 0) return 0;
    const int n = p.rcount[it.bh * p.NQB + it.j];
    return max(1, min(n, p.NQB - it.j));
}

// Item of this CTA's round r, or -1 past the end: the items sorted by
// decreasing step count (dkv_order_kernel) are dealt to the CTAs in snake
// order (forward on even rounds, backward on odd ones), so every CTA gets
// about the same number of steps although a key block is attended by one to
// hundreds of query blocks.
__device__ __forceinline__ int item_at(const Params& p, int r) {
    const int g = (int)gridDim.x;
    const long long pos = (long long)r * g + ((r & 1) ? g - 1 - (int)blockIdx.x : (int)blockIdx.x);
    return pos < p.n_items ? __ldg(p.order + pos) : -1;
}

// What a softmax thread needs for step m of item (b, h, j): the query block,
// the gate of block j in that block's selection, and its row's LSE and Dr.
// The reverse-list entry of a step is loaded two steps ahead and the loads
// that depend on it one step ahead, all independent of each other (no load
// address waits on another load's value inside a step).
struct StepMeta {
    bool cur, in_range, row_ok;
    int slot, idxv;
    float lg, lse, drow;
};
__device__ __forceinline__ StepMeta step_meta(const Params& p, int ent, const KItem& it, int m, int row) {
    StepMeta s;
    const int t = m % p.ntile;
    const int j = it.j;
    int i = ent >> 16;
    s.slot = ent & 0xFFFF;
    s.in_range = i >= j && i < p.NQB;
    if (!s.in_range) i = j;
    s.cur = (i == j);
    const long long sidx = (it.bh * p.NQB + i) * p.K + min(s.slot, p.K - 1);
    s.idxv = s.cur ? j : __ldg(p.idx + sidx);
    s.lg = s.cur ? 0.f : __ldg(p.log_gate + sidx);
    const int hs = 2 * t + (row >> 6);
    // rows of an absent head, or past the sequence's end, contribute nothing
    s.row_ok = hs < p.G && i * 64 + (row & 63) < it.len;
    const int hq = it.h * p.G + (hs < p.G ? hs : 0);
    const long long lrow = ((long long)it.b * p.Hq + hq) * p.S + (long long)i * 64 + (row & 63);
    s.lse = s.row_ok ? __ldg(p.lse + lrow) : 0.f;
    s.drow = s.row_ok ? __ldg(p.Dr + lrow) : 0.f;
    return s;
}

__global__ void __launch_bounds__(kThreads, 1)
dkv_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
           const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &bars->abort;
    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        mbar_init(&bars->kv_empty, 2);                  // the S and dP warps
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->o_full[s], 1);
            mbar_init(&bars->slot_empty[s], 1);         // the tile's last reader (dK^T or dV^T warp)
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->s_full[b], 2);
            mbar_init(&bars->tm_free[b], 256);
        }
        mbar_init(&bars->pds_full, 256);                // dS written
        mbar_init(&bars->pds_empty, 1);                 // dS read (the dK^T warp)
        mbar_init(&bars->p_full, 256);                  // P written
        mbar_init(&bars->p_empty, 1);                   // P read (the dV^T warp)
        mbar_init(&bars->acc_full, 2);
        mbar_init(&bars->acc_empty, 256);
        for (int w = 0; w < 4; ++w) mbar_init(&bars->drain[w], 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t s_base = smem_u32(smem);

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0) {
            uint32_t item_it = 0, g = 0, npos = 0;      // npos: Q / dO tiles issued
            bool kv_issued = false;
            for (int r = 0, id; (id = item_at(p, r)) >= 0 && !*abort; ++r) {
                const KItem it = item_of(p, id);
                const int n = n_entries(p, it);
                if (n == 0) continue;                   // key block past the sequence's end
                const int h = it.h, j = it.j;
                if (!mbar_wait(&bars->kv_empty, (item_it & 1) ^ 1, abort, p.status)) break;
                ++item_it;
                mbar_expect_tx(&bars->kv_full, 4 * kBox);
                for (int a = 0; a < 2; ++a) {
                    tma_load_3d(smem + kOffK + a * kBlkAtom, &map_k, &bars->kv_full, a * 64, h, (int)(it.start + j * 64));
                    tma_load_3d(smem + kOffV + a * kBlkAtom, &map_v, &bars->kv_full, a * 64, h, (int)(it.start + j * 64));
                }
                kv_issued = true;
                const int32_t* list = p.rlist + (it.bh * p.NQB + j) * p.NQB;
                bool ok = true;
                for (int e = 0; e < n && ok; ++e) {
                    int i = __ldg(list + e) >> 16;
                    if (i < j || i >= p.NQB) {
                        flag_status(p.status, kStatusBadData);
                        i = j;
                    }
                    for (int t = 0; t < p.ntile && ok; ++t, ++g) {
                        // Q of step g, then its dO, each into the next ring slot
                        for (int part = 0; part < 2 && ok; ++part) {
                            const uint32_t pos = 2 * g + part;
                            const int sl = pos % kSlots;
                            if (!(ok = mbar_wait(&bars->slot_empty[sl], ((pos / kSlots) & 1) ^ 1, abort, p.status))) break;
                            uint64_t* fb = part == 0 ? &bars->q_full[sl] : &bars->o_full[sl];
                            const CUtensorMap* mp = part == 0 ? &map_q : &map_do;
                            mbar_expect_tx(fb, 4 * kBox);
                            for (int s = 0; s < 2; ++s) {
                                const int hs = 2 * t + s;
                                const int hq = h * p.G + (hs < p.G ? hs : 0);
                                for (int a = 0; a < 2; ++a)
                                    tma_load_3d(smem + kOffRing + sl * kTile + a * kTileAtom + s * kBox, mp, fb, a * 64,
                                                hq, (int)(it.start + i * 64));
                            }
                            ++npos;
                        }
                    }
                }
                if (!ok) break;
            }
            if (*abort) {           // let every copy in flight land before the CTA exits
                volatile int no_abort = 0;
                for (uint32_t pos = npos > (uint32_t)kSlots ? npos - kSlots : 0u; pos < npos; ++pos) {
                    const uint32_t gg = pos / 2;
                    mbar_wait(pos & 1 ? &bars->o_full[pos % kSlots] : &bars->q_full[pos % kSlots], (gg / kSlots) & 1,
                              &no_abort, nullptr);
                }
                if (kv_issued) mbar_wait(&bars->kv_full, (item_it - 1) & 1, &no_abort, nullptr);
            }
        }
    } else if (is_issuer_warp(warp)) {
        // ----------------------------------------------------- issuing warps
        const int slot = issuer_slot(warp);             // 0: S, 1: dP, 2: dV^T, 3: dK^T
        uint32_t item_it = 0, g = 0;
        bool ok = true;
        if (slot < 2) {
            const bool is_s = slot == 0;
            const uint32_t id_s = idesc_bf16(128, 64, false, false);
            const uint32_t kv_lo = sdesc_lo(s_base + (is_s ? kOffK : kOffV), 16);
            for (int r = 0, id; (id = item_at(p, r)) >= 0 && ok; ++r) {
                const int N = n_entries(p, item_of(p, id)) * p.ntile;
                if (N == 0) continue;                   // key block past the sequence's end
                if (!(ok = mbar_wait_warp(&bars->kv_full, item_it & 1, abort, p.status))) break;
                ++item_it;
                for (int m = 0; m < N && ok; ++m, ++g) {
                    const uint32_t pos = 2 * g + (is_s ? 0 : 1);
                    const int sl = pos % kSlots;
                    if (!(ok = mbar_wait_warp(is_s ? &bars->q_full[sl] : &bars->o_full[sl], (g / kSlots) & 1, abort,
                                              p.status)))
                        break;
                    // both warpgroups have read the previous S / dP of this buffer out of TMEM
                    const int buf = g & 1;
                    if (g >= 2 && !(ok = mbar_wait_warp(&bars->tm_free[buf], ((g - 2) >> 1) & 1, abort, p.status)))
                        break;
                    tc_fence_after();
                    const uint32_t a_lo = sdesc_lo(s_base + kOffRing + sl * kTile, 16);   // K-major Q / dO
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t ao = (kk >> 2) * kTileAtom + (kk & 3) * 32;
                        const uint32_t bo = (kk >> 2) * kBlkAtom + (kk & 3) * 32;
                        mma_ss_e(tmem + 128 * buf + (is_s ? 0u : 64u), a_lo + (ao >> 4), kHi, kv_lo + (bo >> 4), kHi,
                                 id_s, kk > 0);
                    }
                    mma_commit_e(&bars->s_full[buf]);
                }
                if (!ok) break;
                mma_commit_e(&bars->kv_empty);          // K_j / V_j may be replaced
            }
        } else {
            // dV^T += dO^T P (slot 2) or dK^T += Q^T dS (slot 3): A = the step's dO / Q
            // tile MN-major, B = P / dS MN-major
            const bool is_v = slot == 2;
            const uint32_t id_t = idesc_bf16(128, 64, true, true);
            const uint32_t acc = tmem + (is_v ? kTmAccV : kTmAccK);
            const uint32_t pb_lo = sdesc_lo(s_base + (is_v ? kOffP : kOffDS), kRowTile);
            for (int r = 0, id; (id = item_at(p, r)) >= 0 && ok; ++r) {
                const int N = n_entries(p, item_of(p, id)) * p.ntile;
                if (N == 0) continue;                   // key block past the sequence's end
                // the drain of the previous item has read the accumulators
                if (!(ok = mbar_wait_warp(&bars->acc_empty, (item_it & 1) ^ 1, abort, p.status))) break;
                ++item_it;
                for (int m = 0; m < N && ok; ++m, ++g) {
                    if (!(ok = mbar_wait_warp(is_v ? &bars->p_full : &bars->pds_full, g & 1, abort, p.status))) break;
                    tc_fence_after();
                    const int sl = (2 * g + (is_v ? 1 : 0)) % kSlots;
                    const uint32_t at_lo = sdesc_lo(s_base + kOffRing + sl * kTile, kTileAtom);   // MN-major
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss_e(acc, at_lo + ((kk * 2048) >> 4), kHi, pb_lo + ((kk * 2048) >> 4), kHi, id_t,
                                 (m > 0 || kk > 0) ? 1u : 0u);
                    mma_commit_e(&bars->slot_empty[sl]);   // the tile's last reader
                    mma_commit_e(is_v ? &bars->p_empty : &bars->pds_empty);
                }
                if (!ok) break;
                mma_commit_e(&bars->acc_full);
            }
        }
        mma_commit_e(&bars->drain[slot]);
        volatile int no_abort = 0;
        mbar_wait(&bars->drain[slot], 0, &no_abort, nullptr);
    } else {
        // ------------------------------------------------ softmax warpgroups
        const int w = (warp - 2) >> 2;                  // keys [32 w, 32 w + 32) of every step
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int r_in = row & 63;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        uint8_t* bufP = smem + kOffP;
        uint8_t* bufS = smem + kOffDS;
        uint32_t item_it = 0, g = 0;
        bool ok = true;
        for (int r = 0, id; (id = item_at(p, r)) >= 0 && ok; ++r) {
            const KItem it = item_of(p, id);
            const int N = n_entries(p, it) * p.ntile;
            if (N == 0) continue;                       // key block past the sequence's end
            const int j = it.j;
            const int32_t* list = p.rlist + (it.bh * p.NQB + j) * p.NQB;
            // metadata pipeline: entry of step m + 2 and loads of step m + 1 in flight
            int ent2 = (1 < N) ? __ldg(list + 1 / p.ntile) : 0;
            StepMeta nxt = step_meta(p, __ldg(list), it, 0, row);
            for (int m = 0; m < N; ++m, ++g) {
                const StepMeta sm = nxt;
                if (m + 1 < N) nxt = step_meta(p, ent2, it, m + 1, row);
                if (m + 2 < N) ent2 = __ldg(list + (m + 2) / p.ntile);
                const int buf = g & 1;
                if (!(ok = mbar_wait(&bars->s_full[buf], (g >> 1) & 1, abort, p.status))) break;
                tc_fence_after();
                const bool valid = sm.in_range && (sm.cur || (sm.slot < p.K && sm.idxv == j));
                // log2 domain; rows of an absent head (or a bad entry) get -inf: P = dS = 0
                const float off = (valid && sm.row_ok) ? sm.lg * kLog2e - sm.lse * kLog2e : -INFINITY;
                const float drs = sm.drow * p.sm_scale;
                uint32_t sv[32], pv[32];
                const uint32_t tS = tmem + lane_base + 128 * buf + 32 * w;
                tmem_ld32(tS, sv);
                tmem_ld32(tS + 64, pv);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&bars->tm_free[buf]);       // S/dP columns may be refilled
                // P first, so that dV^T += dO^T P (and the release of the dO slot) starts
                // while dS is computed; each tile is rewritten once its MMA of the
                // previous step has read it
                unsigned long long pr[16];              // P of the half's keys, in pairs
                if (g > 0 && !(ok = mbar_wait(&bars->p_empty, (g - 1) & 1, abort, p.status))) break;
                {
                    const unsigned long long sc2 = f2_pack(p.scale2, p.scale2), off2 = f2_pack(off, off);
                    const int lim = sm.cur ? r_in : 63;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t pp[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int e = 8 * c + 2 * e2;
                            float2 x = f2_unpack(
                                f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, off2));
                            if (sm.cur) {
                                x.x = (32 * w + e > lim) ? -INFINITY : x.x;
                                x.y = (32 * w + e + 1 > lim) ? -INFINITY : x.y;
                            }
                            const float p0 = fast_exp2(x.x), p1 = fast_exp2(x.y);
                            pr[4 * c + e2] = f2_pack(p0, p1);
                            pp[e2] = pack_bf16x2(p0, p1);
                        }
                        *reinterpret_cast<uint4*>(bufP + sw128_offset(row, 4 * w + c)) =
                            make_uint4(pp[0], pp[1], pp[2], pp[3]);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars->p_full);
                if (g > 0 && !(ok = mbar_wait(&bars->pds_empty, (g - 1) & 1, abort, p.status))) break;
                {
                    const unsigned long long sm2 = f2_pack(p.sm_scale, p.sm_scale), nd2 = f2_pack(-drs, -drs);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t dd[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int e = 8 * c + 2 * e2;
                            const unsigned long long dp =
                                f2_fma(f2_pack(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1])), sm2, nd2);
                            const float2 d = f2_unpack(f2_mul(pr[4 * c + e2], dp));
                            dd[e2] = pack_bf16x2(d.x, d.y);
                        }
                        *reinterpret_cast<uint4*>(bufS + sw128_offset(row, 4 * w + c)) =
                            make_uint4(dd[0], dd[1], dd[2], dd[3]);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars->pds_full);
            }
            if (!ok) break;
            // drain: warpgroup 0 writes dV, warpgroup 1 writes dK (TMEM lane = head-dim index);
            // keys past the sequence's end are not stored
            if (!(ok = mbar_wait(&bars->acc_full, item_it & 1, abort, p.status))) break;
            ++item_it;
            tc_fence_after();
            {
                const int d = row;
                const int keys = min(64, it.len - j * 64);
                __nv_bfloat16* out = (w == 0 ? p.dv : p.dk) + (it.start + (long long)j * 64) * p.Hkv * kD +
                                     (long long)it.h * kD + d;
                const long long key_stride = (long long)p.Hkv * kD;
#pragma unroll 1
                for (int qt = 0; qt < 4; ++qt) {
                    uint32_t v0[16];
                    tmem_ld16(tmem + lane_base + (w == 0 ? kTmAccV : kTmAccK) + 16 * qt, v0);
                    tmem_wait_ld();
                    __nv_bfloat16* o2 = out + 16 * qt * key_stride;
                    if (16 * qt + 16 <= keys) {
#pragma unroll
                        for (int u = 0; u < 16; ++u) o2[u * key_stride] = __float2bfloat16_rn(__uint_as_float(v0[u]));
                    } else {
#pragma unroll
                        for (int u = 0; u < 16; ++u)
                            if (16 * qt + u < keys) o2[u * key_stride] = __float2bfloat16_rn(__uint_as_float(v0[u]));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->acc_empty);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace dkv

// ================================================================ helpers
// Dr = rowsum(O * dO) over D = 128 for every (token, hq) row; Dr as [B, Hq, S]
// (rows of no sequence are skipped). HBM-bound: a warp takes 8 consecutive
// rows, 16 lanes per row with 16-byte loads, all eight loads of a lane issued
// before any is used.
constexpr int kDotRowsPerWarp = 8;
__global__ void __launch_bounds__(256) dot_rows_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout, long long rows, int B,
                                                       int S, int Hq, const int32_t* __restrict__ cu,
                                                       float* __restrict__ Dr) {
    const long long w0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kDotRowsPerWarp;
    const int lane = threadIdx.x & 31, half = lane >> 4, l16 = lane & 15;
    uint4 a[kDotRowsPerWarp / 2], c[kDotRowsPerWarp / 2];
#pragma unroll
    for (int r = 0; r < kDotRowsPerWarp / 2; ++r) {
        const long long row = w0 + 2 * r + half;
        a[r] = c[r] = make_uint4(0u, 0u, 0u, 0u);
        if (row < rows) {
            a[r] = __ldg(reinterpret_cast<const uint4*>(o + row * kD) + l16);
            c[r] = __ldg(reinterpret_cast<const uint4*>(dout + row * kD) + l16);
        }
    }
#pragma unroll
    for (int r = 0; r < kDotRowsPerWarp / 2; ++r) {
        const uint32_t* x = reinterpret_cast<const uint32_t*>(&a[r]);
        const uint32_t* y = reinterpret_cast<const uint32_t*>(&c[r]);
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = bf16x2_to_f32(x[q]), g = bf16x2_to_f32(y[q]);
            acc = fmaf(f.x, g.x, fmaf(f.y, g.y, acc));
        }
#pragma unroll
        for (int m = 8; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
        const long long row = w0 + 2 * r + half;
        int b, t;
        if (l16 == 0 && row < rows && token_seq(cu, B, S, row / Hq, b, t)) {
            const int hq = (int)(row % Hq);
            Dr[((long long)b * Hq + hq) * S + t] = acc;
        }
    }
}

// Orders the dk/dv items (b, h, j): head by head (b, h ascending, so the CTAs
// working at the same time share one head's Q/dO in L2), and inside a head by
// decreasing step count (the length of block j's reverse list, `bpb` buckets
// of equal width per head), so that the snake deal in dkv_kernel balances the
// CTAs. Counted per bucket, scanned by one warp, scattered; the order inside
// a bucket is arbitrary (every item is computed on its own, so results do not
// depend on it).
constexpr int kOrderMaxBuckets = 8192;
__global__ void __launch_bounds__(1024) dkv_order_kernel(const int32_t* __restrict__ rcount, int n, int NQB, int bpb,
                                                         int32_t* __restrict__ order) {
    __shared__ int cnt[kOrderMaxBuckets];
    const int nb = (n / NQB) * bpb;
    for (int c = threadIdx.x; c < nb; c += blockDim.x) cnt[c] = 0;
    __syncthreads();
    auto bucket = [&](int id) {
        const int j = id % NQB, bh = id / NQB;
        const int c = max(1, min(rcount[id], NQB - j));      // steps of item id, 1..NQB
        return bh * bpb + (bpb - 1) - (int)((long long)(c - 1) * bpb / NQB);
    };
    for (int id = threadIdx.x; id < n; id += blockDim.x) atomicAdd(&cnt[bucket(id)], 1);
    __syncthreads();
    if (threadIdx.x < 32) {                                   // exclusive scan: lane l owns a chunk of buckets
        const int l = threadIdx.x, per = (nb + 31) / 32, lo = min(nb, l * per), hi = min(nb, lo + per);
        int sum = 0;
        for (int c = lo; c < hi; ++c) sum += cnt[c];
        int incl = sum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, d);
            if (l >= d) incl += t;
        }
        int run = incl - sum;
        for (int c = lo; c < hi; ++c) {
            const int v = cnt[c];
            cnt[c] = run;
            run += v;
        }
    }
    __syncthreads();
    for (int id = threadIdx.x; id < n; id += blockDim.x) order[atomicAdd(&cnt[bucket(id)], 1)] = id;
}

__global__ void rev_fill_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int rows, int NQB,
                                int K, int Hkv, const int32_t* __restrict__ cu, int S, long long T,
                                int16_t* __restrict__ slotmap) {
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int i = (int)(row % NQB);
    const long long bh = row / NQB;
    const int len = seq_range(cu, (int)(bh / Hkv), S, T, nullptr).len;
    const int c = i * 64 < len ? max(0, min(cnt[row], min(K, i))) : 0;
    for (int k = lane; k < c; k += 32) {
        const int j = idx[row * K + k];
        if (j >= 0 && j < i) slotmap[(bh * NQB + j) * NQB + i] = (int16_t)(k + 1);
    }
}

__global__ void rev_list_kernel(const int16_t* __restrict__ slotmap, int rows, int NQB, int32_t* __restrict__ rlist,
                                int32_t* __restrict__ rcount) {
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);   // (bh, j)
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int j = (int)(row % NQB);
    int32_t* list = rlist + row * NQB;
    const int16_t* sm = slotmap + row * NQB;
    if (lane == 0) list[0] = (j << 16) | 0xFFFF;
    int n = 1;
    for (int i0 = j + 1; i0 < NQB; i0 += 32) {
        const int i = i0 + lane;
        const int v = (i < NQB) ? sm[i] : 0;
        const unsigned ball = __ballot_sync(0xffffffffu, v != 0);
        if (v != 0) list[n + __popc(ball & ((1u << lane) - 1u))] = (i << 16) | (v - 1);
        n += __popc(ball);
    }
    if (lane == 0) rcount[row] = n;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Ws {
    float* Dr;
    float* gsum;
    int16_t* slotmap;
    int32_t* rlist;
    int32_t* rcount;
    int32_t* order;
};

Ws carve(void* w, int B, int S, int Hq, int Hkv, int K) {
    const int NQB = (S + 63) / 64;
    char* p = static_cast<char*>(w);
    Ws r;
    r.Dr = reinterpret_cast<float*>(p);
    p += align256(sizeof(float) * (size_t)B * Hq * S);
    r.gsum = reinterpret_cast<float*>(p);
    p += align256(sizeof(float) * (size_t)B * Hkv * NQB * (size_t)(K > 0 ? K : 1));
    r.slotmap = reinterpret_cast<int16_t*>(p);
    p += align256(sizeof(int16_t) * (size_t)B * Hkv * NQB * NQB);
    r.rlist = reinterpret_cast<int32_t*>(p);
    p += align256(sizeof(int32_t) * (size_t)B * Hkv * NQB * NQB);
    r.rcount = reinterpret_cast<int32_t*>(p);
    p += align256(sizeof(int32_t) * (size_t)B * Hkv * NQB);
    r.order = reinterpret_cast<int32_t*>(p);
    return r;
}

}  // namespace

size_t bwd_sm100_workspace(int B, int S, int Hq, int Hkv, int K) {
    const int NQB = (S + 63) / 64;
    return align256(sizeof(float) * (size_t)B * Hq * S) +
           align256(sizeof(float) * (size_t)B * Hkv * NQB * (size_t)(K > 0 ? K : 1)) +
           align256(sizeof(int16_t) * (size_t)B * Hkv * NQB * NQB) +
           align256(sizeof(int32_t) * (size_t)B * Hkv * NQB * NQB) + 2 * align256(sizeof(int32_t) * (size_t)B * Hkv * NQB);
}

cudaError_t launch_bwd_sm100(const BwdArgs& bw, cudaStream_t st) {
    const AttnArgs& a = bw.a;
    const int NQB = (a.S + 63) / 64, G = a.Hq / a.Hkv;
    const long long rows = a.T;
    CUtensorMap mq, mdo, mk, mv;
    if (!make_head_map(&mq, a.q, rows, a.Hq, kD) || !make_head_map(&mdo, bw.dout, rows, a.Hq, kD) ||
        !make_head_map(&mk, a.k, rows, a.Hkv, kD) || !make_head_map(&mv, a.v, rows, a.Hkv, kD))
        return cudaErrorInvalidValue;
    Ws ws = carve(bw.workspace, a.B, a.S, a.Hq, a.Hkv, a.K);
    cudaError_t e;
    const int bhq = a.B * a.Hkv * NQB;
    if ((e = cudaMemsetAsync(ws.gsum, 0, sizeof(float) * (size_t)bhq * (a.K > 0 ? a.K : 1), st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(ws.slotmap, 0, sizeof(int16_t) * (size_t)bhq * NQB, st)) != cudaSuccess) return e;
    const long long drows = rows * a.Hq;
    const long long dwarps = (drows + kDotRowsPerWarp - 1) / kDotRowsPerWarp;
    dot_rows_kernel<<<(unsigned)((dwarps + 7) / 8), 256, 0, st>>>(
        (const __nv_bfloat16*)bw.o, (const __nv_bfloat16*)bw.dout, drows, a.B, a.S, a.Hq, a.cu, ws.Dr);
    rev_fill_kernel<<<(bhq + 7) / 8, 256, 0, st>>>(a.idx, a.cnt, bhq, NQB, a.K, a.Hkv, a.cu, a.S, a.T, ws.slotmap);
    rev_list_kernel<<<(bhq + 7) / 8, 256, 0, st>>>(ws.slotmap, bhq, NQB, ws.rlist, ws.rcount);
    // buckets per head: 64, fewer when there are more than 128 (batch, KV head) pairs
    const int n_bh = a.B * a.Hkv;
    const int bpb = n_bh * 64 <= kOrderMaxBuckets ? 64 : (n_bh <= kOrderMaxBuckets ? kOrderMaxBuckets / n_bh : 0);
    if (bpb == 0) return cudaErrorInvalidValue;
    dkv_order_kernel<<<1, 1024, 0, st>>>(ws.rcount, bhq, NQB, bpb, ws.order);
    count_launches(4);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    Params p;
    p.B = a.B;
    p.S = a.S;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.G = G;
    p.K = a.K;
    p.NQB = NQB;
    p.cu = a.cu;
    p.T = a.T;
    p.ntile = (G + 1) / 2;
    p.idx = a.idx;
    p.cnt = a.cnt;
    p.log_gate = a.log_gate;
    p.lse = bw.lse;
    p.Dr = ws.Dr;
    p.rlist = ws.rlist;
    p.rcount = ws.rcount;
    p.order = ws.order;
    p.scale2 = a.sm_scale * kLog2e;
    p.sm_scale = a.sm_scale;
    p.inv_scale = 1.f / a.sm_scale;
    p.dq = static_cast<__nv_bfloat16*>(bw.dq);
    p.dk = static_cast<__nv_bfloat16*>(bw.dk);
    p.dv = static_cast<__nv_bfloat16*>(bw.dv);
    p.gsum = ws.gsum;
    p.status = a.status;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

    p.n_items = a.B * a.Hkv * NQB * p.ntile;
    if ((e = cudaFuncSetAttribute(dqk::dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dqk::kSmem)) !=
        cudaSuccess)
        return e;
    dqk::dq_kernel<<<p.n_items < sms ? p.n_items : sms, dqk::kThreadsDq, dqk::kSmem, st>>>(mq, mdo, mk, mv, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    p.n_items = a.B * a.Hkv * NQB;
    if ((e = cudaFuncSetAttribute(dkv::dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dkv::kSmem)) !=
        cudaSuccess)
        return e;
    dkv::dkv_kernel<<<p.n_items < sms ? p.n_items : sms, kThreads, dkv::kSmem, st>>>(mq, mdo, mk, mv, p);
    count_launches(2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_ds_finalize(bw.s, bw.ld_s, bw.lse_s, a.idx, a.cnt, ws.gsum, a.B, a.Hkv, NQB, a.K, a.cu, a.S, a.T,
                              bw.ds, st);
}

}  // namespace sas
