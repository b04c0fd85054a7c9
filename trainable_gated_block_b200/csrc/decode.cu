// sas_decode_paged: one gated block-sparse decode step over a paged KV cache.
//
// SAS review (paper.oopus.info) §2.3, eq. o_SAS and §2.4: the query of
// sequence n (position kv_len-1) attends its current block c with gate 1 and
// its kept history blocks with their log-gates; §2.6: the KV cache lives in
// 64-token pages. Only the kept pages are read: each (page, KV head) is one
// contiguous 16 KiB tile of K and one of V.
//
// HBM-bound design. Work item = (sequence n, KV head h) with its cnt + 1
// blocks; the items' blocks are laid end to end ((K + 1) slots per item) and
// cut into one contiguous range per CTA, so every SM streams the same number
// of blocks. One persistent CTA per SM:
//  * a producer warp resolves 32 slots at a time (selection entry -> page ->
//    gate, in parallel over its lanes) and TMA-copies each kept (page, head)
//    K and V tile, 128-byte swizzled, into a ring of six 32 KiB stages;
//  * three consumer warps take the CTA's blocks round robin (warp w owns
//    stages w and w + 3, so each warp's stages are double buffered). A warp
//    does a whole block on the tensor cores with mma.sync m16n8k16: the G
//    query heads of the group are the rows of the 16-row A operand (the
//    rest zero), S = Q K^T over 64 keys (8 n-tiles x 8 k-steps), then an
//    online softmax in the log2 domain on the S fragments (a row lives in
//    the 4 lanes of a quad), then O += P V (16 n-tiles x 4 k-steps) with P
//    taken straight from the S fragments. K and V fragments come from shared
//    memory by ldmatrix (conflict-free on the swizzled layout);
//  * when the CTA leaves an item, the warps' states are merged through
//    shared memory into one partial (m, l, o) for that (item, CTA).
// A combine kernel merges the (at most a few) partials of each query head.
// The tensor work is tiny (the kernel is bound by HBM); using it keeps the
// per-block instruction count low enough that the math hides under the
// page reads.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace sas {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kWarps = 3;                          // consumer warps
constexpr int kThreads = (kWarps + 1) * 32;        // + one producer warp
constexpr int kStages = 2 * kWarps;                // warp w owns stages w and w + kWarps
constexpr uint32_t kBoxBytes = 64 * 128;           // TMA box: 64 rows x 64 dims (128 B)
constexpr int kShortRows = 8;                      // short box (one 128-byte swizzle period) for a partial block
constexpr uint32_t kShortBytes = kShortRows * 128;
constexpr uint32_t kTileBytes = 2 * kBoxBytes;     // one (page, head) tile of K or V
constexpr uint32_t kStageBytes = 2 * kTileBytes;
constexpr uint32_t kOffMo = kStages * kStageBytes;                 // merge scratch: o [warp][8][D]
constexpr uint32_t kOffMl = kOffMo + kWarps * 8 * kD * 4;          // merge scratch: m, l [warp][8][2]
constexpr uint32_t kOffMeta = kOffMl + kWarps * 8 * 2 * 4;         // per-stage (bias, valid keys)
constexpr uint32_t kOffBar = kOffMeta + kStages * 8;
constexpr uint32_t kSmem = kOffBar + 2 * kStages * 8 + 16 + 1024;  // + alignment slack
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");

struct Params {
    const __nv_bfloat16* q;
    int num_pages;
    const int32_t* page_table;
    int max_pages;
    const int32_t* kv_len;
    int Hq, Hkv, G, K;
    const int32_t* idx;
    const int32_t* cnt;
    const float* log_gate;
    float qscale;           // sm_scale * log2(e)
    long long V;            // n_items * (K + 1) block slots
    int grid;
    int nslot;              // partial slots per query head
    float* part_o;          // [N * Hq, nslot, D]
    float* part_ml;         // [N * Hq, nslot, 2]
    int* status;
};

// CTA c owns block slots [c V / grid, (c + 1) V / grid); cta_of is its inverse.
__host__ __device__ __forceinline__ long long slot_begin(long long c, long long V, int grid) { return c * V / grid; }
__host__ __device__ __forceinline__ int cta_of(long long s, long long V, int grid) {
    return (int)(((s + 1) * grid - 1) / V);
}

struct ItemInfo {
    int n, h, L, c, n_sel;
    bool ok;
};
__device__ __forceinline__ ItemInfo item_info(const Params& p, int item, bool flag) {
    ItemInfo r;
    r.n = item / p.Hkv;
    r.h = item % p.Hkv;
    r.L = p.kv_len[r.n];
    r.ok = r.L >= 1 && r.L <= p.max_pages * kBlock;
    r.c = r.ok ? (r.L - 1) / kBlock : 0;
    int n_sel = p.cnt[item];
    const int hi = min(p.K, r.c);
    if (n_sel < 0 || n_sel > hi) {
        if (flag) flag_status(p.status, kStatusBadData);
        n_sel = max(0, min(n_sel, hi));
    }
    r.n_sel = n_sel;
    if (!r.ok && flag) flag_status(p.status, kStatusBadData);
    return r;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, rows 8..15 zero: only a0a1 / a4a5 given) * B (16x8 bf16)
__device__ __forceinline__ void mma_rows8(float (&d)[4], uint32_t a01, uint32_t a45, uint32_t b01, uint32_t b23) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a01), "r"(0u), "r"(a45), "r"(0u), "r"(b01), "r"(b23));
}

// Byte offset of 16-byte chunk `c` (0..15 over the 128 dims) of row `r` in a
// tile stored as two 64-row x 128-byte boxes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
    return (uint32_t)(c >> 3) * kBoxBytes + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
              const __grid_constant__ CUtensorMap map_k8, const __grid_constant__ CUtensorMap map_v8, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* mo = reinterpret_cast<float*>(smem + kOffMo);
    float* ml = reinterpret_cast<float*>(smem + kOffMl);
    float2* meta = reinterpret_cast<float2*>(smem + kOffMeta);   // (bias log2 units, valid keys)
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* empty = full + kStages;
    int* abort_flag = reinterpret_cast<int*>(empty + kStages);
    volatile int* abort = abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const long long v0 = slot_begin(blockIdx.x, p.V, p.grid), v1 = slot_begin(blockIdx.x + 1, p.V, p.grid);
    const int Kp1 = p.K + 1;
    // the combine kernel may be scheduled now (it waits for this grid to finish)
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;");

    if (warp == kWarps) {
        // ----------------------------------------------------------- producer
        // The 32 lanes resolve 32 block slots at a time (selection entry, page,
        // gate: dependent loads, done in parallel); lane 0 then issues the
        // copies of the kept ones in slot order. The next batch is resolved
        // once the ring is full, while its copies are in flight, so the ring
        // does not drain during those loads.
        if (lane == 0) {
            prefetch_tensormap(&map_k);
            prefetch_tensormap(&map_v);
            prefetch_tensormap(&map_k8);
            prefetch_tensormap(&map_v8);
        }
        struct Slot {
            bool use;
            int row0;
            float bias, nvalid;
        };
        auto resolve = [&](long long base) {
            const long long v = base + lane;
            Slot s{false, -1, 0.f, 0.f};
            if (v < v1) {
                const int item = (int)(v / Kp1), t = (int)(v % Kp1);
                const ItemInfo inf = item_info(p, item, true);
                if (inf.ok && t <= inf.n_sel) {
                    s.use = true;
                    const bool cur = (t == inf.n_sel);
                    const long long srow = (long long)item * p.K + t;
                    const int j = cur ? inf.c : p.idx[srow];
                    int page = -1;
                    if (j >= 0 && (cur || j < inf.c) && j < p.max_pages)
                        page = p.page_table[(long long)inf.n * p.max_pages + j];
                    const bool ok = page >= 0 && page < p.num_pages;
                    if (!ok) flag_status(p.status, kStatusBadData);
                    s.bias = cur ? 0.f : p.log_gate[srow] * kLog2e;
                    s.nvalid = ok ? (float)(cur ? inf.L - inf.c * kBlock : kBlock) : 0.f;
                    s.row0 = ok ? (page * p.Hkv + inf.h) * kBlock : -1;   // < 2^31 (checked on the host)
                }
            }
            return s;
        };
        uint32_t it = 0;
        bool ok_run = true;
        Slot cur = resolve(v0);
        for (long long base = v0; base < v1 && ok_run; base += 32) {
            const bool more = base + 32 < v1;
            Slot nxt{false, -1, 0.f, 0.f};
            bool resolved = !more;
            int issued = 0;
            unsigned todo = __ballot_sync(0xffffffffu, cur.use);
            while (todo) {
                const int b = __ffs(todo) - 1;
                todo &= todo - 1;
                const int rb = __shfl_sync(0xffffffffu, cur.row0, b);
                const float bb = __shfl_sync(0xffffffffu, cur.bias, b);
                const float nb = __shfl_sync(0xffffffffu, cur.nvalid, b);
                if (lane == 0) {
                    const int st = it % kStages;
                    if (!mbar_wait(&empty[st], ((it / kStages) & 1) ^ 1, abort, p.status)) {
                        ok_run = false;
                    } else {
                        meta[st] = make_float2(bb, nb);
                        uint8_t* dst = smem + st * kStageBytes;
                        const int nv = (int)nb;
                        if (rb >= 0 && nv < kBlock) {
                            // partial block (the current one): only the 8-row groups holding tokens
                            const int ng = (nv + kShortRows - 1) / kShortRows;
                            mbar_expect_tx(&full[st], (uint32_t)ng * 4 * kShortBytes);
                            for (int g8 = 0; g8 < ng; ++g8)
                                for (int a = 0; a < 2; ++a) {
                                    const uint32_t off = a * kBoxBytes + g8 * kShortBytes;
                                    tma_load_3d(dst + off, &map_k8, &full[st], a * 64, 0, rb + g8 * kShortRows);
                                    tma_load_3d(dst + kTileBytes + off, &map_v8, &full[st], a * 64, 0,
                                                rb + g8 * kShortRows);
                                }
                        } else if (rb >= 0) {
                            mbar_expect_tx(&full[st], kStageBytes);
                            for (int a = 0; a < 2; ++a) {
                                tma_load_3d(dst + a * kBoxBytes, &map_k, &full[st], a * 64, 0, rb);
                                tma_load_3d(dst + kTileBytes + a * kBoxBytes, &map_v, &full[st], a * 64, 0, rb);
                            }
                        } else {
                            mbar_arrive(&full[st]);
                        }
                        ++it;
                    }
                }
                ok_run = __shfl_sync(0xffffffffu, ok_run, 0);
                if (!ok_run) break;
                if (!resolved && ++issued == kStages) {
                    nxt = resolve(base + 32);
                    resolved = true;
                }
            }
            if (!resolved) nxt = resolve(base + 32);
            cur = nxt;
        }
        if (lane == 0 && *abort) {       // let the copies in flight land before the CTA exits
            volatile int no_abort = 0;
            const uint32_t lo = it > (uint32_t)kStages ? it - kStages : 0;
            for (uint32_t k = lo; k < it; ++k) mbar_wait(&full[k % kStages], (k / kStages) & 1, &no_abort, nullptr);
        }
        return;   // the producer takes no part in the consumers' named barrier
    }

    // -------------------------------------------------------------- consumers
    const int grp = lane >> 2, tig = lane & 3;     // mma fragment coordinates: row (head), column pair
    const uint32_t s_base = smem_u32(smem);
    uint32_t qa[8][2];          // Q as A fragments: 8 k-steps x (dims 2tig.., 8+2tig..) of head grp
    float o[16][4];             // O accumulators: 16 n-tiles of 8 dims (rows 8..15 stay 0)
    float m = -INFINITY, l = 0.f;   // this thread's head: running max (log2) and its partial sum
    uint32_t blk = 0;           // blocks of this CTA's stream seen so far
    int cur_item = -1;
    ItemInfo inf{};
    bool dead = false;

    auto flush = [&]() {
        // row sum over the quad, then every warp's state to shared memory
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
            *reinterpret_cast<float2*>(mo + (warp * 8 + grp) * kD + 8 * nt + 2 * tig) = make_float2(o[nt][0], o[nt][1]);
        if (tig == 0) {
            ml[(warp * 8 + grp) * 2] = m;
            ml[(warp * 8 + grp) * 2 + 1] = l;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
        const int slot = (int)blockIdx.x - cta_of((long long)cur_item * Kp1, p.V, p.grid);
        for (int e = threadIdx.x; e < p.G * kD; e += kWarps * 32) {
            const int g = e / kD, d = e % kD;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) M = fmaxf(M, ml[(w * 8 + g) * 2]);
            float acc = 0.f, L = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    const float mw = ml[(w * 8 + g) * 2];
                    const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
                    acc = fmaf(mo[(w * 8 + g) * kD + d], f, acc);
                    L = fmaf(ml[(w * 8 + g) * 2 + 1], f, L);
                }
            }
            const long long row = ((long long)inf.n * p.Hq + inf.h * p.G + g) * p.nslot + slot;
            p.part_o[row * kD + d] = acc;
            if (d == 0) {
                p.part_ml[row * 2] = M;
                p.part_ml[row * 2 + 1] = L;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
    };

    for (long long v = v0; v < v1; ++v) {
        const int item = (int)(v / Kp1), t = (int)(v % Kp1);
        if (item != cur_item) {
            if (cur_item >= 0) flush();
            cur_item = item;
            inf = item_info(p, item, false);
            const bool real = grp < p.G;
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
                p.q + ((long long)inf.n * p.Hq + inf.h * p.G + (real ? grp : 0)) * kD);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                qa[kk][0] = real ? __ldg(qrow + 8 * kk + tig) : 0u;
                qa[kk][1] = real ? __ldg(qrow + 8 * kk + 4 + tig) : 0u;
            }
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
            m = -INFINITY;
            l = 0.f;
        }
        if (!inf.ok || t > inf.n_sel) continue;
        const uint32_t b = blk++;
        if (b % kWarps != (uint32_t)warp || dead) continue;      // another warp's block
        const int st = b % kStages;
        if (!mbar_wait_warp(&full[st], (b / kStages) & 1, abort, p.status)) {
            dead = true;              // keep walking the slots so the flush barriers still meet
            continue;
        }
        const float2 md = meta[st];
        const int nvalid = (int)md.y;
        if (nvalid > 0) {
            const uint32_t kt = s_base + st * kStageBytes, vt = kt + kTileBytes;
            // S = Q K^T: n-tile nt = keys 8nt..8nt+7; ldmatrix.x4 gives B fragments of two n-tiles
            float s[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    const int key = 16 * np + 8 * (lane >> 4) + (lane & 7);
                    const int chunk = 2 * kk + ((lane >> 3) & 1);
                    uint32_t bf[4];
                    ldsm_x4(kt + tile_off(key, chunk), bf);
                    mma_rows8(s[2 * np], qa[kk][0], qa[kk][1], bf[0], bf[1]);
                    mma_rows8(s[2 * np + 1], qa[kk][0], qa[kk][1], bf[2], bf[3]);
                }
            }
            // online softmax for head grp over keys 8nt + 2tig + {0, 1}
            float bm = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int key = 8 * nt + 2 * tig + e;
                    const float x = key < nvalid ? fmaf(s[nt][e], p.qscale, md.x) : -INFINITY;
                    s[nt][e] = x;
                    bm = fmaxf(bm, x);
                }
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
            const float mn = fmaxf(m, bm);
            const float sc = mn == -INFINITY ? 1.f : exp2f(m - mn);
            m = mn;
            uint32_t pa[8];             // P as A fragments: n-tile nt -> keys 8nt + 2tig..
            float ls = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const float p0 = mn == -INFINITY ? 0.f : exp2f(s[nt][0] - mn);
                const float p1 = mn == -INFINITY ? 0.f : exp2f(s[nt][1] - mn);
                ls += p0 + p1;
                pa[nt] = pack_bf16x2(p0, p1);
            }
            l = fmaf(l, sc, ls);
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                o[nt][0] *= sc;
                o[nt][1] *= sc;
            }
            if (nvalid < kBlock) {
                // rows past the sequence end (the current block) are zeroed: their p
                // is 0, but whatever the page holds there must not reach O as 0 * NaN
                uint8_t* vrow = smem + st * kStageBytes + kTileBytes;
                for (int e = nvalid * 16 + lane; e < kBlock * 16; e += 32)
                    *reinterpret_cast<uint4*>(vrow + tile_off(e >> 4, e & 15)) = make_uint4(0u, 0u, 0u, 0u);
                fence_proxy_async_smem();     // ordered before the stage's next TMA refill
                __syncwarp();
            }
            // O += P V: k-step kk = keys 16kk..16kk+15; ldmatrix.x4.trans gives B of two n-tiles
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    const int key = 16 * kk + 8 * ((lane >> 3) & 1) + (lane & 7);
                    const int chunk = 2 * np + (lane >> 4);
                    uint32_t bf[4];
                    ldsm_x4_t(vt + tile_off(key, chunk), bf);
                    mma_rows8(o[2 * np], pa[2 * kk], pa[2 * kk + 1], bf[0], bf[1]);
                    mma_rows8(o[2 * np + 1], pa[2 * kk], pa[2 * kk + 1], bf[2], bf[3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (cur_item >= 0) flush();
}

__global__ void __launch_bounds__(kD)
decode_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml, int nslot, int Hq, int Hkv,
                      int G, int K, long long V, int grid, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
    // launched as a programmatic dependent of decode_kernel: its blocks may be
    // resident before the decode grid ends; wait for that grid's writes here
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const long long row = blockIdx.x;          // n * Hq + hq
    const int d = threadIdx.x;
    const long long n = row / Hq;
    const int hq = (int)(row % Hq);
    const long long item = n * Hkv + hq / G;
    const long long s0 = item * (K + 1);
    const int nsl = cta_of(s0 + K, V, grid) - cta_of(s0, V, grid) + 1;
    const float* ml = part_ml + row * nslot * 2;
    float M = -INFINITY;
    for (int s = 0; s < nsl; ++s) M = fmaxf(M, ml[2 * s]);
    float Lsum = 0.f, acc = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < nsl; ++s) {
            const float w = exp2f(ml[2 * s] - M);     // 0 for empty partials (m = -inf)
            Lsum = fmaf(ml[2 * s + 1], w, Lsum);
            acc = fmaf(part_o[(row * nslot + s) * kD + d], w, acc);
        }
    }
    o[row * kD + d] = __float2bfloat16_rn(acc / Lsum);
    if (lse != nullptr && d == 0) lse[row] = (M + log2f(Lsum)) * kLn2;
}

struct Layout {
    long long V;
    int grid, nslot;
};
Layout layout(int N, int Hkv, int K) {
    Layout r;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    r.V = (long long)N * Hkv * (K + 1);
    r.grid = (int)(r.V < sms ? r.V : sms);
    if (r.grid < 1) r.grid = 1;
    const long long mn = r.V / r.grid;                       // shortest CTA range
    const long long span = (K + 1 + mn - 1) / mn + 1;        // CTAs one item's slots can touch
    r.nslot = (int)(span < r.grid ? span : r.grid);
    return r;
}

}  // namespace

size_t decode_workspace(int N, int Hq, int Hkv, int D, int K) {
    (void)D;
    const Layout lay = layout(N, Hkv, K);
    const size_t per = (size_t)N * Hq * lay.nslot;
    return sizeof(float) * (per * kD + per * 2);
}

cudaError_t launch_decode(const DecodeArgs& a, void* workspace, cudaStream_t st) {
    const int G = a.Hq / a.Hkv;
    if (G < 1 || G > 8 || a.Hq % a.Hkv) return cudaErrorInvalidValue;
    const long long cache_rows = (long long)a.num_pages * a.Hkv * kBlock;
    if (cache_rows > 0x7fffffffLL) return cudaErrorInvalidValue;   // TMA row coordinates are int32
    const Layout lay = layout(a.N, a.Hkv, a.K);
    float* part_o = static_cast<float*>(workspace);
    float* part_ml = part_o + (size_t)a.N * a.Hq * lay.nslot * kD;
    CUtensorMap mk, mv, mk8, mv8;
    if (!make_head_map(&mk, a.k_cache, cache_rows, 1, kD) || !make_head_map(&mv, a.v_cache, cache_rows, 1, kD) ||
        !make_head_map(&mk8, a.k_cache, cache_rows, 1, kD, kShortRows) ||
        !make_head_map(&mv8, a.v_cache, cache_rows, 1, kD, kShortRows))
        return cudaErrorInvalidValue;
    Params p;
    p.q = (const __nv_bfloat16*)a.q;
    p.num_pages = a.num_pages;
    p.page_table = a.page_table;
    p.max_pages = a.max_pages;
    p.kv_len = a.kv_len;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.G = G;
    p.K = a.K;
    p.idx = a.idx;
    p.cnt = a.cnt;
    p.log_gate = a.log_gate;
    p.qscale = a.sm_scale * kLog2e;
    p.V = lay.V;
    p.grid = lay.grid;
    p.nslot = lay.nslot;
    p.part_o = part_o;
    p.part_ml = part_ml;
    p.status = a.status;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    decode_kernel<<<lay.grid, kThreads, kSmem, st>>>(mk, mv, mk8, mv8, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // programmatic dependent launch: the combine's blocks are placed while the
    // decode grid drains, which removes the launch gap between the two kernels
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.N * a.Hq));
    cfg.blockDim = dim3(kD);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_combine_kernel, (const float*)part_o, (const float*)part_ml, lay.nslot, a.Hq,
                           a.Hkv, G, a.K, lay.V, lay.grid, (__nv_bfloat16*)a.o, a.lse);
    if (e != cudaSuccess) return e;
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace sas
