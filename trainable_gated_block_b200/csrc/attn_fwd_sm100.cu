// Gated block-sparse causal attention forward on the sm_100a tensor cores.
//
// SAS review (paper.oopus.info) §2.3, eq. o_SAS: o = softmax(q K_S^T + log g_S) V_S
// over the current block (gate 1, causal) and the kept history blocks (gate
// g_m = exp(s_m - LSE(s)), §2.4), computed tile by tile without the full
// logit matrix (§2.6). bf16 operands, fp32 accumulation, D = 128.
//
// Work item = (batch b, KV head h, query block i, head group tg): up to two
// 128-row Q tiles, each tile = 2 query heads x the 64 rows of block i. All
// query heads of a GQA group share the kept blocks, so one K/V block feeds
// both Q tiles. Persistent grid; items head by head, longest first within a head.
// Sequence b occupies token rows start_b .. start_b + len_b - 1 (a dense batch,
// or a packed batch of different lengths). Its last block may be partial: the
// Q box reads past the sequence (those rows are computed and dropped), and the
// keys past its end lie above every valid row, so the causal mask removes
// them. Items of query blocks past a sequence's end are skipped by every role.
//
// One step = one kept block (64 keys). Warp roles (352 threads):
//   warp 0      TMA producer: the Q tiles once per item, then K and V of one
//               block per step into a 4-stage ring (128B-swizzled).
//   warps 1, 10 tcgen05 issuers (one thread each), warp 1 for Q tile 0 (and
//               TMEM owner), warp 10 for tile 1: a single thread issues MMAs
//               at a bounded rate, so each tile has its own. S_t = Q_t K^T
//               into one of two S buffers per tile, O_t += P_t V with P read
//               from TMEM. S of step j+2 is issued as soon as PV of step j is,
//               so the softmax of step j+1 never waits for an MMA. On an
//               item with one Q tile the idle issuer still waits for each Q
//               and K/V phase and releases it, so it never falls two phases
//               behind those barriers.
//   warps 2-5   softmax of Q tile 0, warps 6-9 of tile 1: one row per thread
//               (one TMEM lane); logits = sm_scale q.k + log-gate in the log2
//               domain, causal mask on the diagonal block, running max/sum;
//               P (bf16) over the consumed S buffer; O in TMEM rescaled only
//               when the max grows by more than 2^8 (the only point, besides
//               the end of the item, where the softmax waits for a PV: the
//               issuer publishes completed PVs as a count); final o and LSE.
// TMEM (512 columns): tile t owns [256t, 256t+256): S buffers at +0 and +64
// (64 columns each, P overwrites the first 32), O at +128.
#include "launch.h"
#include "sm100.cuh"

namespace sas {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kNS = 4;                              // K/V stages (one block each)
constexpr int kThreads = 352;
constexpr int kIssuer1Warp = 10;                  // MMA issuer of Q tile 1
constexpr uint32_t kBox = 64 * 128;                 // one TMA box: 64 rows x 128 B
constexpr uint32_t kQAtom = 2 * kBox;               // 128 rows x 128 B
constexpr uint32_t kQTile = 2 * kQAtom;             // 128 rows x 256 B
constexpr uint32_t kBlkAtom = kBox;                 // 64 keys x 128 B
constexpr uint32_t kBlk = 2 * kBlkAtom;             // 64 keys x 256 B
constexpr uint32_t kStage = 2 * kBlk;               // K block + V block
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = 2 * kQTile;                         // 64 KB
constexpr uint32_t kOffBar = kOffKV + kNS * kStage;             // 192 KB
constexpr uint32_t kSmemBytes = kOffBar + 1024 + 1024;
constexpr float kRescaleThreshold = 8.0f;           // log2 units

struct Meta {            // one block of an item's list
    int j;               // block index actually loaded
    float bias2;         // log-gate * log2(e) (0 on the current block)
    int live;            // 0: masked out entirely (bad index)
    int cur;             // 1: the query's own block (causal mask)
};

struct Bars {
    uint64_t q_full, q_empty;
    uint64_t k_full[kNS], v_full[kNS], kv_empty[kNS];
    uint64_t s_full[2][2], p_full[2][2];
    uint64_t o_done[2], o_empty[2];
    uint64_t drain[2];
    uint32_t tmem_base;
    int abort;
    uint32_t pv_count[2];    // PVs of tile t known complete (issuer writes, softmax polls)
};

// Bounded wait until the published count reaches `target` (acquire); gives up
// like mbar_wait: on the abort flag or after about kWaitCycles clocks.
__device__ __forceinline__ bool wait_count(const uint32_t* c, uint32_t target, volatile int* abort, int* status) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(c)) : "memory");
    if ((int)(v - target) >= 0) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(c)) : "memory");
        if ((int)(v - target) >= 0) return true;
        if ((it & 63u) == 0) {
            if (*abort) return false;
            if (clock64() - t0 > kWaitCycles) {
                *abort = 1;
                flag_status(status, kStatusTimeout);
                return false;
            }
        }
    }
}

struct Params {
    int B, S, Hq, Hkv, G, K, NQB, ntg, n_items;
    const int32_t* cu;                  // packed sequence bounds [B + 1], or nullptr (dense)
    long long T;                        // token rows of q/k/v
    const int32_t* idx;
    const int32_t* cnt;
    const float* log_gate;
    float scale2;                       // sm_scale * log2(e)
    __nv_bfloat16* o;
    float* lse;
    int* status;
};

struct Item {
    int b, h, i, tg, nt, c, nb, len;
    long long row, start;               // selection row; first token row of the sequence
    bool skip;                          // query block past the sequence's end
};

__device__ __forceinline__ Item item_of(const Params& p, int id) {
    Item it;
    // head by head (the CTAs working at the same time share one head's K/V in
    // L2), query blocks from the last (longest items) down, then the head group
    const int per_bh = p.NQB * p.ntg;
    const int bh = id / per_bh, r = id % per_bh;
    it.i = p.NQB - 1 - r / p.ntg;
    it.tg = r % p.ntg;
    it.h = bh % p.Hkv;
    it.b = bh / p.Hkv;
    it.nt = (4 * it.tg + 2 < p.G) ? 2 : 1;
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

// Block k of the item's list: kept blocks ascending, then the current block.
// An out-of-range index is replaced by the current block, fully masked.
__device__ __forceinline__ Meta meta_at(const Params& p, const Item& it, int k) {
    Meta m;
    if (k < it.c) {
        const int j = __ldg(p.idx + it.row * p.K + k);
        const bool ok = j >= 0 && j < it.i;
        m.j = ok ? j : it.i;
        m.bias2 = ok ? __ldg(p.log_gate + it.row * p.K + k) * kLog2e : 0.f;
        m.live = ok;
        m.cur = 0;
    } else {
        m.j = it.i;
        m.bias2 = 0.f;
        m.live = 1;
        m.cur = 1;
    }
    return m;
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
        mbar_init(&bars->q_empty, 2);                   // one arrival per MMA issuer
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->kv_empty[s], 2);
        }
        for (int t = 0; t < 2; ++t) {
            for (int b = 0; b < 2; ++b) {
                mbar_init(&bars->s_full[t][b], 1);
                mbar_init(&bars->p_full[t][b], 128);
            }
            mbar_init(&bars->o_done[t], 1);
            mbar_init(&bars->o_empty[t], 128);
        }
        mbar_init(&bars->drain[0], 1);
        mbar_init(&bars->drain[1], 1);
        bars->abort = 0;
        bars->pv_count[0] = bars->pv_count[1] = 0;
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
    const uint32_t sKV = smem_u32(smem + kOffKV);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kv_it = 0, q_it = 0;
            int last_it[kNS] = {-1, -1, -1, -1};
            bool q_issued = false;
            if (p.cu != nullptr)           // check the packed bounds once (flags a bad sequence)
                for (int b = 0; b < p.B; ++b) seq_range(p.cu, b, p.S, p.T, p.status);
            for (int id = live_item(p, blockIdx.x); id < p.n_items && !*abort; id = live_item(p, id + gridDim.x)) {
                const Item it = item_of(p, id);
                if (p.cnt[it.row] != it.c) flag_status(p.status, kStatusBadData);
                if (!mbar_wait(&bars->q_empty, (q_it & 1) ^ 1, abort, p.status)) break;
                mbar_expect_tx(&bars->q_full, (uint32_t)it.nt * 4 * kBox);
                for (int t = 0; t < it.nt; ++t)
                    for (int s = 0; s < 2; ++s) {
                        const int slot = 4 * it.tg + 2 * t + s;
                        const int hq = it.h * p.G + (slot < p.G ? slot : 0);
                        for (int a = 0; a < 2; ++a)
                            tma_load_3d(smem + kOffQ + t * kQTile + a * kQAtom + s * kBox, &map_q, &bars->q_full,
                                        a * 64, hq, (int)(it.start + it.i * 64));
                    }
                q_issued = true;
                ++q_it;
                for (int k = 0; k < it.nb; ++k, ++kv_it) {
                    const int st = kv_it % kNS;
                    if (!mbar_wait(&bars->kv_empty[st], ((kv_it / kNS) & 1) ^ 1, abort, p.status)) break;
                    const Meta m = meta_at(p, it, k);
                    if (!m.live) flag_status(p.status, kStatusBadData);
                    mbar_expect_tx(&bars->k_full[st], 2 * kBox);
                    for (int a = 0; a < 2; ++a)
                        tma_load_3d(smem + kOffKV + st * kStage + a * kBlkAtom, &map_k, &bars->k_full[st], a * 64,
                                    it.h, (int)(it.start + m.j * 64));
                    mbar_expect_tx(&bars->v_full[st], 2 * kBox);
                    for (int a = 0; a < 2; ++a)
                        tma_load_3d(smem + kOffKV + st * kStage + kBlk + a * kBlkAtom, &map_v, &bars->v_full[st],
                                    a * 64, it.h, (int)(it.start + m.j * 64));
                    last_it[st] = (int)kv_it;
                }
            }
            if (*abort) {
                volatile int no_abort = 0;
                for (int s = 0; s < kNS; ++s)
                    if (last_it[s] >= 0) {
                        const uint32_t par = ((uint32_t)last_it[s] / kNS) & 1;
                        mbar_wait(&bars->k_full[s], par, &no_abort, nullptr);
                        mbar_wait(&bars->v_full[s], par, &no_abort, nullptr);
                    }
                if (q_issued) mbar_wait(&bars->q_full, (q_it - 1) & 1, &no_abort, nullptr);
            }
        }
    } else if (warp == 1 || warp == kIssuer1Warp) {
        // ------------------------------------------------------------ MMA issuers, one per Q tile
        // (one thread issues tcgen05.mma at a bounded rate, so each tile has its own)
        if (lane == 0) {
            const int t = (warp == 1) ? 0 : 1;
            const uint32_t id_s = idesc_bf16(128, 64, false, false);
            const uint32_t id_pv = idesc_bf16(128, kD, false, true);
            uint32_t kv_it = 0, q_it = 0, p_it[2] = {0, 0}, oe_it = 0, pv_n = 0;
            constexpr uint32_t kHi = sdesc_hi(1024);
            const uint32_t q_lo = sdesc_lo(sQ + t * kQTile, 16);
            auto issue_s = [&](int st, int buf) {
                const uint32_t k_lo = sdesc_lo(sKV + st * kStage, 16);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t ao = (kk >> 2) * kQAtom + (kk & 3) * 32;
                    const uint32_t bo = (kk >> 2) * kBlkAtom + (kk & 3) * 32;
                    mma_ss_w(tmem + 256 * t + 64 * buf, q_lo + (ao >> 4), kHi, k_lo + (bo >> 4), kHi, id_s, kk > 0);
                }
                mma_commit(&bars->s_full[t][buf]);
            };
            bool ok = true;
            for (int id = live_item(p, blockIdx.x); id < p.n_items && ok; id = live_item(p, id + gridDim.x)) {
                const Item it = item_of(p, id);
                if (!(ok = mbar_wait(&bars->q_full, q_it & 1, abort, p.status))) break;
                ++q_it;
                if (t >= it.nt) {
                    // Tile 1 idle: still wait every phase of the shared Q and K/V barriers and
                    // release it at once, so that this issuer never falls two phases behind (a
                    // parity wait on a barrier two phases ahead would pass on the wrong phase).
                    for (int k = 0; k < it.nb && ok; ++k, ++kv_it) {
                        const int st = kv_it % kNS;
                        const uint32_t par = (kv_it / kNS) & 1;
                        if (!(ok = mbar_wait(&bars->k_full[st], par, abort, p.status) &&
                                   mbar_wait(&bars->v_full[st], par, abort, p.status)))
                            break;
                        if (k + 1 == it.nb) mbar_arrive(&bars->q_empty);
                        mbar_arrive(&bars->kv_empty[st]);
                    }
                    continue;
                }
                tc_fence_after();
                // prologue: S of the first two steps
                for (int k = 0; k < 2 && k < it.nb && ok; ++k) {
                    const uint32_t g = kv_it + k;
                    if (!(ok = mbar_wait(&bars->k_full[g % kNS], (g / kNS) & 1, abort, p.status))) break;
                    tc_fence_after();
                    issue_s(g % kNS, k & 1);
                }
                if (!ok) break;
                if (it.nb <= 2) mma_commit(&bars->q_empty);
                for (int k = 0; k < it.nb && ok; ++k, ++kv_it) {
                    const int st = kv_it % kNS;
                    const int buf = k & 1;
                    if (!(ok = mbar_wait(&bars->v_full[st], (kv_it / kNS) & 1, abort, p.status))) break;
                    if (!(ok = mbar_wait(&bars->p_full[t][buf], p_it[buf] & 1, abort, p.status))) break;
                    ++p_it[buf];
                    if (k == 0) {
                        if (!(ok = mbar_wait(&bars->o_empty[t], (oe_it & 1) ^ 1, abort, p.status))) break;
                        ++oe_it;
                    }
                    tc_fence_after();
                    const uint32_t v_lo = sdesc_lo(sKV + st * kStage + kBlk, kBlkAtom);   // MN-major V
                    const uint32_t acc0 = k > 0 ? 1u : 0u;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts_w(tmem + 256 * t + 128, tmem + 256 * t + 64 * buf + kk * 8, v_lo + ((kk * 2048) >> 4),
                                 kHi, id_pv, kk > 0 ? 1u : acc0);
                    mma_commit(&bars->o_done[t]);
                    if (k + 2 < it.nb) {
                        const uint32_t g2 = kv_it + 2;
                        if (!(ok = mbar_wait(&bars->k_full[g2 % kNS], (g2 / kNS) & 1, abort, p.status))) break;
                        tc_fence_after();
                        issue_s(g2 % kNS, buf);
                    }
                    if (k + 3 == it.nb) mma_commit(&bars->q_empty);
                    mma_commit(&bars->kv_empty[st]);
                    // publish PV completion: the softmax waits for it only when it
                    // rescales O and at the end of the item
                    if (!(ok = mbar_wait(&bars->o_done[t], pv_n & 1, abort, p.status))) break;
                    ++pv_n;
                    asm volatile("st.release.cta.shared.u32 [%0], %1;" ::"r"(smem_u32(&bars->pv_count[t])), "r"(pv_n)
                                 : "memory");
                }
            }
            mma_commit(&bars->drain[t]);
            volatile int no_abort = 0;
            mbar_wait(&bars->drain[t], 0, &no_abort, nullptr);
        }
    } else if (warp >= 2 && warp < 10) {
        // ------------------------------------------------------------ softmax / epilogue
        const int t = (warp - 2) >> 2;                  // Q tile of this warpgroup
        const int quarter = warp & 3;                   // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;            // row of the Q tile = TMEM lane
        const int slot_in_tile = row >> 6, r_in = row & 63;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tT = tmem + lane_base + 256 * t;
        const uint32_t tO = tT + 128;
        // pv_count[t]: PVs of this tile completed so far (published by the issuer)
        uint32_t s_it[2] = {0, 0}, pv_it = 0;
        for (int id = live_item(p, blockIdx.x); id < p.n_items; id = live_item(p, id + gridDim.x)) {
            const Item it = item_of(p, id);
            if (t >= it.nt) continue;
            const int slot = 4 * it.tg + 2 * t + slot_in_tile;
            float m_ref = -INFINITY, l = 0.f;
            bool ok = true;
            Meta nxt = meta_at(p, it, 0);
            for (int k = 0; k < it.nb; ++k) {
                const int buf = k & 1;
                const Meta m = nxt;
                if (k + 1 < it.nb) nxt = meta_at(p, it, k + 1);    // prefetch the next block's gate
                if (!(ok = mbar_wait(&bars->s_full[t][buf], s_it[buf] & 1, abort, p.status))) break;
                ++s_it[buf];
                tc_fence_after();
                uint32_t raw[2][32];
                tmem_ld32(tT + 64 * buf, raw[0]);
                tmem_ld32(tT + 64 * buf + 32, raw[1]);
                tmem_wait_ld();
                // logit (log2 units) = S * scale2 + bias2. On a block without masked
                // keys the row max is taken over the raw S (the affine map is monotonic,
                // so the maximum is the same number) and each P costs one FMA and one
                // exp2; on the diagonal or a flagged block the masked logits replace S
                // in place and the same FMA runs with scale 1.
                const bool masked = m.cur || !m.live;
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // 4 independent chains
                float mx, sc, bias;
                if (masked) {
#pragma unroll
                    for (int u = 0; u < 64; ++u) {
                        const bool live = m.live && u <= r_in;
                        const float x = live ? fmaf(__uint_as_float(raw[u >> 5][u & 31]), p.scale2, m.bias2) : -INFINITY;
                        raw[u >> 5][u & 31] = __float_as_uint(x);
                        mx4[u & 3] = fmaxf(mx4[u & 3], x);
                    }
                    mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                    sc = 1.f;
                    bias = 0.f;
                } else {
                    float r;                             // the S that gives the largest logit
                    if (p.scale2 >= 0.f) {
#pragma unroll
                        for (int u = 0; u < 64; u += 2)     // two keys per three-input max
                            mx4[(u >> 1) & 3] = max3(mx4[(u >> 1) & 3], __uint_as_float(raw[u >> 5][u & 31]),
                                                     __uint_as_float(raw[(u + 1) >> 5][(u + 1) & 31]));
                        r = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                    } else {
                        float mn4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
#pragma unroll
                        for (int u = 0; u < 64; ++u) mn4[u & 3] = fminf(mn4[u & 3], __uint_as_float(raw[u >> 5][u & 31]));
                        r = fminf(fminf(mn4[0], mn4[1]), fminf(mn4[2], mn4[3]));
                    }
                    mx = fmaf(r, p.scale2, m.bias2);
                    sc = p.scale2;
                    bias = m.bias2;
                }
                const float m_new = fmaxf(m_ref, mx);
                const bool need = m_new > m_ref + kRescaleThreshold;
                const bool rescale = __any_sync(0xffffffffu, need) && k > 0;    // warp-uniform
                const float f = need ? exp2f(m_ref - m_new) : 1.f;                // O and l scale
                if (need) {
                    l *= f;
                    m_ref = m_new;
                }
                const float c = bias - ((m_ref == -INFINITY) ? 0.f : m_ref);   // P = 2^(S sc + c)
                uint32_t pk[32];
                // two keys per f32x2 instruction: the FMA and the running sums
                const unsigned long long sc2 = f2_pack(sc, sc), c2 = f2_pack(c, c);
                unsigned long long l2[4] = {0ull, 0ull, 0ull, 0ull};     // 4 independent chains of pairs
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int u = 2 * e;
                    const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(raw[u >> 5][u & 31]),
                                                              __uint_as_float(raw[(u + 1) >> 5][(u + 1) & 31])),
                                                      sc2, c2));
                    const float p0 = fast_exp2(x.x), p1 = fast_exp2(x.y);
                    l2[e & 3] = f2_add(l2[e & 3], f2_pack(p0, p1));
                    pk[e] = pack_bf16x2(p0, p1);
                }
                {
                    const float2 a0 = f2_unpack(f2_add(l2[0], l2[1])), a1 = f2_unpack(f2_add(l2[2], l2[3]));
                    l += (a0.x + a0.y) + (a1.x + a1.y);
                }
                tmem_st32(tT + 64 * buf, pk);
                if (rescale) {
                    // O is rescaled in TMEM: PV of the previous step must be complete
                    if (!(ok = wait_count(&bars->pv_count[t], pv_it + k, abort, p.status))) break;
                    tc_fence_after();
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
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[t][buf]);
            }
            if (!ok) break;
            if (!wait_count(&bars->pv_count[t], pv_it + it.nb, abort, p.status)) break;
            pv_it += it.nb;
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const bool store = slot < p.G && it.i * 64 + r_in < it.len;
            const int hq = it.h * p.G + slot;
            const long long orow = (it.start + (long long)it.i * 64 + r_in) * p.Hq + hq;
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

}  // namespace

cudaError_t launch_fwd_sm100(const AttnArgs& a, void* o, float* lse, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    const long long rows = a.T;
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
    p.NQB = (a.S + 63) / 64;
    p.cu = a.cu;
    p.T = a.T;
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
