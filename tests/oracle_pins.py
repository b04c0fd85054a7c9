"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each ``pin_*`` takes the oracle module as an argument, so the same pins can
be run against deliberately broken copies of it (``test_oracle_pins.py``
plants such mistakes on the CPU and checks that some pin catches each one).

Sources of truth used here:
* a hand-worked example (``golden/q0_worked_example.json``),
* closed forms: with K >= #history and equal scores the method is dense
  causal attention with history logits shifted by -ln(#history); with K = 0
  it is block-diagonal causal attention (SAS review (paper.oopus.info),
  §2.3 eq. o_SAS and §2.4 eq. log g),
* library routines: torch's scaled_dot_product_attention (fp64, CPU) with an
  additive mask, scipy's logsumexp,
* the rank definition of Top-K with the lower-index tie-break,
* brute force with Python loops on tiny inputs,
* central finite differences in fp64,
* invariants: shift invariance in s, exact zero influence of unselected K/V,
  rows of ds sum to zero, probabilities sum to one, causality (a sequence
  cut inside a block gives the first rows of the longer sequence).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F
from scipy.special import logsumexp as sp_logsumexp

HERE = os.path.dirname(os.path.abspath(__file__))
BLOCK = 64


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _sdpa(q_rows, keys, vals, bias, scale):
    """torch SDPA in fp64 on one head: q_rows [T,D], keys/vals [U,D], bias [T,U]."""
    q_t = torch.from_numpy(np.ascontiguousarray(q_rows))[None, None]
    k_t = torch.from_numpy(np.ascontiguousarray(keys))[None, None]
    v_t = torch.from_numpy(np.ascontiguousarray(vals))[None, None]
    m_t = torch.from_numpy(np.ascontiguousarray(bias))[None, None]
    return F.scaled_dot_product_attention(q_t, k_t, v_t, attn_mask=m_t, scale=scale)[0, 0].numpy()


def _rank_select(row, K):
    """Top-K by the rank definition: j is kept iff #{better} < K, where m beats
    j when s_m > s_j, or s_m == s_j and m < j."""
    n = len(row)
    out = []
    for j in range(n):
        rank = sum(1 for m in range(n) if row[m] > row[j]) + sum(1 for m in range(j) if row[m] == row[j])
        if rank < K:
            out.append(j)
    return out


# ---------------------------------------------------------------------------
def pin_topk_rank(O):
    r = np.random.default_rng(11)
    for trial in range(400):
        nh = int(r.integers(0, 48))
        K = int(r.integers(0, 14))
        if trial % 3 == 0:
            row = r.choice(np.array([-1.5, -0.0, 0.0, 0.25, 2.0, 3.0]), size=nh)
        elif trial % 3 == 1:
            row = np.full(nh, 0.625)
        else:
            row = r.standard_normal(nh).astype(np.float32).astype(np.float64)
        assert O.topk_history(row, nh, K) == _rank_select(list(row), K), (trial, row, K)


def pin_select_gates(O):
    s = _rand((2, 3, 11, 11), 12).astype(np.float32)
    K = 4
    idx, cnt, lg, lse_s = O.select(s, K, O.prefill_history(11))
    for b in range(2):
        for h in range(3):
            for i in range(11):
                row = s[b, h, i, :i].astype(np.float64)
                assert cnt[b, h, i] == min(K, i)
                sel = _rank_select(list(row), K)
                assert list(idx[b, h, i, :cnt[b, h, i]]) == sel
                assert np.all(idx[b, h, i, cnt[b, h, i]:] == -1)
                assert np.all(np.isneginf(lg[b, h, i, cnt[b, h, i]:]))
                if i == 0:
                    assert np.isneginf(lse_s[b, h, i])
                    continue
                ref = sp_logsumexp(row)
                assert abs(lse_s[b, h, i] - ref) <= 1e-13 * max(1.0, abs(ref))
                gates = lg[b, h, i, :cnt[b, h, i]]
                assert np.allclose(gates, row[sel] - ref, rtol=0, atol=1e-13)
                assert np.all(gates <= 1e-15)
                tot = sp_logsumexp(gates)
                if K >= i:
                    assert abs(tot) <= 1e-13
                else:
                    assert tot < -1e-9


def pin_golden(O):
    with open(os.path.join(HERE, "golden", "q0_worked_example.json")) as f:
        ex = json.load(f)
    inp, exp = ex["inputs"], ex["expect"]
    S, D, K, sc = inp["S"], inp["D"], inp["K"], inp["sm_scale"]
    q = np.zeros((1, S, 1, D))
    k = np.ones((1, S, 1, D))
    v = np.stack([np.arange(S, dtype=np.float64), np.ones(S)], axis=1)[None, :, None, :]
    s = np.array(inp["s"], dtype=np.float64)[None, None]
    idx, cnt, lg, lse_s = O.select(s, K, O.prefill_history(3))
    assert idx[0, 0].tolist() == exp["idx"] and cnt[0, 0].tolist() == exp["cnt"]
    for i in range(3):
        e = exp["log_gate"][i][0]
        assert np.isneginf(lg[0, 0, i, 0]) if e is None else abs(lg[0, 0, i, 0] - e) < 1e-14
        e = exp["lse_s"][i]
        assert np.isneginf(lse_s[0, 0, i]) if e is None else abs(lse_s[0, 0, i] - e) < 1e-14
    o, lse = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    assert np.allclose(o[0, :, 0, 1], exp["o1_all_rows"], rtol=0, atol=1e-12)
    for row in exp["rows"]:
        t = row["t"]
        assert abs(o[0, t, 0, 0] - row["o0_num"] / row["o0_den"]) < 1e-11, (t, o[0, t, 0, 0])
        assert abs(lse[0, 0, t] - math.log(row["lse_arg"])) < 1e-12, t


def _dense_case(seed, S=320, Hq=4, Hkv=2, D=8):
    q = _rand((1, S, Hq, D), seed)
    k = _rand((1, S, Hkv, D), seed + 1)
    v = _rand((1, S, Hkv, D), seed + 2)
    return q, k, v


def pin_dense_equivalence(O):
    """K >= #history and equal scores: dense causal attention, history shifted by -ln(i)."""
    q, k, v = _dense_case(21)
    S, Hq, D = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    NQB = S // BLOCK
    s = np.full((1, k.shape[2], NQB, NQB), 0.7)
    idx, cnt, lg, _ = O.select(s, NQB, O.prefill_history(NQB))
    sc = 1.0 / math.sqrt(D)
    o, _ = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    t = np.arange(S)[:, None]
    u = np.arange(S)[None, :]
    blk = t // BLOCK
    bias = np.where(u <= t, 0.0, -np.inf)
    hist = u < blk * BLOCK
    bias = np.where(hist, -np.log(np.maximum(blk, 1)), bias)
    for hq in range(Hq):
        ref = _sdpa(q[0, :, hq], k[0, :, hq // G], v[0, :, hq // G], bias, sc)
        assert np.allclose(o[0, :, hq], ref, rtol=1e-12, atol=1e-12)


def pin_block_diagonal(O):
    """K = 0: every query attends only the causal part of its own block."""
    q, k, v = _dense_case(31)
    S, Hq, D = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    NQB = S // BLOCK
    s = _rand((1, k.shape[2], NQB, NQB), 32)
    idx, cnt, lg, _ = O.select(s, 0, O.prefill_history(NQB))
    sc = 0.3
    o, _ = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    t = np.arange(S)[:, None]
    u = np.arange(S)[None, :]
    bias = np.where((u <= t) & (u // BLOCK == t // BLOCK), 0.0, -np.inf)
    for hq in range(Hq):
        ref = _sdpa(q[0, :, hq], k[0, :, hq // G], v[0, :, hq // G], bias, sc)
        assert np.allclose(o[0, :, hq], ref, rtol=1e-12, atol=1e-12)


def pin_general_sdpa(O):
    """General Top-K: SDPA with a mask built from the rank selection and scipy gates."""
    q, k, v = _dense_case(41, S=448, Hq=6, Hkv=2, D=8)
    S, Hq, Hkv, D = q.shape[1], q.shape[2], k.shape[2], q.shape[3]
    G = Hq // Hkv
    NQB = S // BLOCK
    s = _rand((1, Hkv, NQB, NQB), 42, 2.0).astype(np.float32)
    K = 3
    idx, cnt, lg, _ = O.select(s, K, O.prefill_history(NQB))
    sc = 1.0 / math.sqrt(D)
    o, lse = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    for h in range(Hkv):
        bias = np.full((S, S), -np.inf)
        for i in range(NQB):
            row = s[0, h, i, :i].astype(np.float64)
            ls = sp_logsumexp(row) if i else 0.0
            for j in _rank_select(list(row), K):
                bias[i * BLOCK:(i + 1) * BLOCK, j * BLOCK:(j + 1) * BLOCK] = row[j] - ls
            for r in range(BLOCK):
                bias[i * BLOCK + r, i * BLOCK:i * BLOCK + r + 1] = 0.0
        for g in range(G):
            hq = h * G + g
            ref = _sdpa(q[0, :, hq], k[0, :, h], v[0, :, h], bias, sc)
            assert np.allclose(o[0, :, hq], ref, rtol=1e-12, atol=1e-12)
            ref_lse = torch.logsumexp(torch.from_numpy(sc * q[0, :, hq] @ k[0, :, h].T + bias), dim=1).numpy()
            assert np.allclose(lse[0, hq], ref_lse, rtol=1e-12, atol=1e-12)


def pin_bruteforce_loops(O):
    """Python loops with math.exp on a tiny case, selection and gates included."""
    S, Hq, Hkv, D, K = 192, 2, 1, 3, 1
    q, k, v = _rand((1, S, Hq, D), 51), _rand((1, S, Hkv, D), 52), _rand((1, S, Hkv, D), 53)
    s = _rand((1, Hkv, 3, 3), 54)
    sc = 0.41
    idx, cnt, lg, _ = O.select(s, K, O.prefill_history(3))
    o, lse = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    for hq in range(Hq):
        for t in range(S):
            i = t // BLOCK
            hist = [float(s[0, 0, i, j]) for j in range(i)]
            keep = {}
            if hist:
                best = max(range(i), key=lambda j: (hist[j], -j))
                mx = max(hist)
                lsum = mx + math.log(sum(math.exp(x - mx) for x in hist))
                keep[best] = hist[best] - lsum
            logits, rows = [], []
            for u in range(S):
                j = u // BLOCK
                if j == i and u <= t:
                    bias = 0.0
                elif j in keep:
                    bias = keep[j]
                else:
                    continue
                dot = sum(q[0, t, hq, d] * k[0, u, 0, d] for d in range(D))
                logits.append(sc * dot + bias)
                rows.append(u)
            mx = max(logits)
            w = [math.exp(x - mx) for x in logits]
            z = sum(w)
            for d in range(D):
                ref = sum(wi * v[0, u, 0, d] for wi, u in zip(w, rows)) / z
                assert abs(o[0, t, hq, d] - ref) < 1e-12
            assert abs(lse[0, hq, t] - (mx + math.log(z))) < 1e-12


def _fd_case():
    S, Hq, Hkv, D, K = 256, 2, 1, 16, 2
    q, k, v = _rand((1, S, Hq, D), 61), _rand((1, S, Hkv, D), 62), _rand((1, S, Hkv, D), 63)
    do = _rand((1, S, Hq, D), 64)
    s = _rand((1, Hkv, 4, 4), 65)
    return q, k, v, do, s, K, 0.25


def _loss(O, q, k, v, s, do, K, sc):
    NQB = q.shape[1] // BLOCK
    idx, cnt, lg, _ = O.select(s, K, O.prefill_history(NQB))
    o, _ = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    return float(np.sum(o * do))


def pin_finite_differences(O):
    q, k, v, do, s, K, sc = _fd_case()
    NQB = 4
    idx, cnt, lg, _ = O.select(s, K, O.prefill_history(NQB))
    dq, dk, dv, ds, _ = O.attn_bwd(q, k, v, do, idx, cnt, lg, s, sc)
    h = 1e-6
    r = np.random.default_rng(66)
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            pos = tuple(int(r.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[pos] += h
            minus[pos] -= h
            args = dict(q=q, k=k, v=v)
            args[name] = plus
            lp = _loss(O, args["q"], args["k"], args["v"], s, do, K, sc)
            args[name] = minus
            lm = _loss(O, args["q"], args["k"], args["v"], s, do, K, sc)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])
    for i in range(1, NQB):
        row = np.sort(s[0, 0, i, :i])
        for j in range(i):
            assert np.all(np.abs(np.diff(row)) > 4 * h) if i > 1 else True
            plus, minus = s.copy(), s.copy()
            plus[0, 0, i, j] += h
            minus[0, 0, i, j] -= h
            fd = (_loss(O, q, k, v, plus, do, K, sc) - _loss(O, q, k, v, minus, do, K, sc)) / (2 * h)
            assert abs(fd - ds[0, 0, i, j]) <= 1e-6 * max(1.0, abs(fd)), (i, j, fd, ds[0, 0, i, j])
    assert np.all(ds[0, 0][np.triu_indices(NQB)] == 0.0)


def pin_shift_invariance(O):
    q, k, v, do, s, K, sc = _fd_case()
    NQB = 4
    a = O.select(s, K, O.prefill_history(NQB))
    b = O.select(s + 3.0, K, O.prefill_history(NQB))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    fin = np.isfinite(a[2])
    assert np.array_equal(fin, np.isfinite(b[2]))
    assert np.allclose(a[2][fin], b[2][fin], rtol=0, atol=1e-13)
    oa, _ = O.attn_fwd(q, k, v, *a[:3], sc)
    ob, _ = O.attn_fwd(q, k, v, *b[:3], sc)
    assert np.allclose(oa, ob, rtol=0, atol=1e-12)
    ga = O.attn_bwd(q, k, v, do, *a[:3], s, sc)
    gb = O.attn_bwd(q, k, v, do, *b[:3], s + 3.0, sc)
    for x, y in zip(ga[:4], gb[:4]):
        assert np.allclose(x, y, rtol=0, atol=1e-11)


def pin_sparsity(O):
    """K/V outside a row's selected blocks and current block have no influence."""
    S, Hq, Hkv, D, K = 512, 2, 1, 8, 2
    q, k, v = _rand((1, S, Hq, D), 71), _rand((1, S, Hkv, D), 72), _rand((1, S, Hkv, D), 73)
    do = _rand((1, S, Hq, D), 74)
    s = _rand((1, Hkv, 8, 8), 75)
    NQB = 8
    idx, cnt, lg, _ = O.select(s, K, O.prefill_history(NQB))
    sc = 0.35
    o, lse = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    for i in range(NQB):
        keep = set(int(j) for j in idx[0, 0, i, :cnt[0, 0, i]]) | {i}
        k2, v2 = k.copy(), v.copy()
        for j in range(NQB):
            if j not in keep:
                k2[0, j * BLOCK:(j + 1) * BLOCK] = _rand((BLOCK, Hkv, D), 100 + j, 5.0)
                v2[0, j * BLOCK:(j + 1) * BLOCK] = _rand((BLOCK, Hkv, D), 200 + j, 5.0)
        o2, lse2 = O.attn_fwd(q, k2, v2, idx, cnt, lg, sc)
        rs = slice(i * BLOCK, (i + 1) * BLOCK)
        assert np.array_equal(o[0, rs], o2[0, rs]) and np.array_equal(lse[0, :, rs], lse2[0, :, rs])
    _, dk, dv, ds, gsum = O.attn_bwd(q, k, v, do, idx, cnt, lg, s, sc)
    picked = set(int(j) for j in idx[0, 0][idx[0, 0] >= 0])
    never = [j for j in range(NQB - 1) if j not in picked]
    assert never, "case should leave some key block unselected"
    for j in never:
        # block j is still attended by its own (diagonal) rows; zero it out of
        # the picture by checking that only the diagonal stripe contributes
        diag_only = O.attn_bwd(q, k, v, do, idx, cnt, lg, s, sc,
                               stripes=[(0, hq, j) for hq in range(Hq)])
        rs = slice(j * BLOCK, (j + 1) * BLOCK)
        assert np.array_equal(dk[0, rs], diag_only[1][0, rs])
        assert np.array_equal(dv[0, rs], diag_only[2][0, rs])
    for i in range(NQB):
        sel = set(int(j) for j in idx[0, 0, i, :cnt[0, 0, i]])
        for j in range(i):
            if j not in sel:
                assert gsum[0, 0, i, j] == 0.0
        assert abs(ds[0, 0, i].sum()) <= 1e-12 * max(1.0, np.abs(ds[0, 0, i]).sum())


def pin_probabilities(O):
    q, k, v = _dense_case(81)
    NQB = q.shape[1] // BLOCK
    s = _rand((1, 2, NQB, NQB), 82)
    idx, cnt, lg, _ = O.select(s, 2, O.prefill_history(NQB))
    q64, k64, v64 = q, k, v
    for hq in range(q.shape[2]):
        for i in range(NQB):
            _, _, P, _ = O.fwd_stripe(q64, k64, v64, idx, cnt, lg, 0.3, 0, hq, i)
            assert np.allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-13)
            assert np.all(P >= 0)


def _paged(kc_rows, vc_rows, n_pages_total, perm_seed):
    """Scatter contiguous [L,Hkv,D] K/V rows of one sequence into 64-token pages."""
    L, Hkv, D = kc_rows.shape
    npg = (L + BLOCK - 1) // BLOCK
    perm = np.random.default_rng(perm_seed).permutation(n_pages_total)[:npg]
    kc = _rand((n_pages_total, Hkv, BLOCK, D), perm_seed + 1)
    vc = _rand((n_pages_total, Hkv, BLOCK, D), perm_seed + 2)
    for p in range(npg):
        rows = slice(p * BLOCK, min(L, (p + 1) * BLOCK))
        n = rows.stop - rows.start
        kc[perm[p], :, :n] = kc_rows[rows].transpose(1, 0, 2)
        vc[perm[p], :, :n] = vc_rows[rows].transpose(1, 0, 2)
    return kc, vc, perm


def pin_decode_vs_sdpa(O):
    Hq, Hkv, D, K = 4, 2, 8, 3
    G = Hq // Hkv
    lens = [1, 64, 65, 200, 640, 700]
    N = len(lens)
    maxp = max((L + 63) // 64 for L in lens)
    q = _rand((N, Hq, D), 91)
    s = _rand((N, Hkv, 16), 92).astype(np.float32)
    kv_len = np.array(lens)
    kcs, vcs, pts, conts = [], [], np.zeros((N, maxp), dtype=np.int64), []
    total = 0
    for n, L in enumerate(lens):
        kr, vr = _rand((L, Hkv, D), 300 + n), _rand((L, Hkv, D), 400 + n)
        kc, vc, perm = _paged(kr, vr, 12, 500 + n)
        kcs.append(kc)
        vcs.append(vc)
        pts[n, :len(perm)] = perm + total
        total += 12
        conts.append((kr, vr))
    kc, vc = np.concatenate(kcs), np.concatenate(vcs)
    idx, cnt, lg, lse_s = O.select(s[:, :, None, :], K, O.decode_history(kv_len)[:, None])
    idx, cnt, lg = idx[:, :, 0], cnt[:, :, 0], lg[:, :, 0]
    sc = 1.0 / math.sqrt(D)
    o, lse = O.decode(q, kc, vc, pts, kv_len, idx, cnt, lg, sc)
    for n, L in enumerate(lens):
        kr, vr = conts[n]
        c = (L - 1) // BLOCK
        for h in range(Hkv):
            row = s[n, h, :c].astype(np.float64)
            bias = np.full((1, L), -np.inf)
            bias[0, c * BLOCK:L] = 0.0
            if c:
                ls = sp_logsumexp(row)
                for j in _rank_select(list(row), K):
                    bias[0, j * BLOCK:(j + 1) * BLOCK] = row[j] - ls
            for g in range(G):
                hq = h * G + g
                ref = _sdpa(q[n, hq][None], kr[:, h], vr[:, h], bias, sc)[0]
                assert np.allclose(o[n, hq], ref, rtol=1e-12, atol=1e-12), (n, hq)


def pin_decode_vs_prefill(O):
    """The last row of a full prefill block equals a decode query at that position."""
    S, Hq, Hkv, D, K = 512, 4, 2, 8, 2
    G = Hq // Hkv
    q, k, v = _rand((1, S, Hq, D), 111), _rand((1, S, Hkv, D), 112), _rand((1, S, Hkv, D), 113)
    NQB = S // BLOCK
    s = _rand((1, Hkv, NQB, NQB), 114)
    sc = 0.3
    idx, cnt, lg, _ = O.select(s, K, O.prefill_history(NQB))
    o, lse = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    kc, vc, perm = _paged(k[0], v[0], 20, 115)
    pt = perm[None]
    kv_len = np.array([S])
    sd = s[:, :, NQB - 1, :].copy()
    didx, dcnt, dlg, _ = O.select(sd[:, :, None, :], K, O.decode_history(kv_len)[:, None])
    od, lsed = O.decode(q[:, S - 1], kc, vc, pt, kv_len, didx[:, :, 0], dcnt[:, :, 0], dlg[:, :, 0], sc)
    assert np.allclose(od[0], o[0, S - 1], rtol=1e-12, atol=1e-12)
    assert np.allclose(lsed[0], lse[0, :, S - 1], rtol=1e-12, atol=1e-12)
    assert G == 2


def pin_standin_scores(O):
    """Stand-in scores against explicit loops, a closed form and their invariances."""
    B, S, Hq, Hkv, D = 2, 192, 6, 2, 8
    G, NQB = Hq // Hkv, S // BLOCK
    q = _rand((B, S, Hq, D), 31)
    k = _rand((B, S, Hkv, D), 32)
    noise = _rand((B, Hkv, NQB, NQB), 33)
    s = O.standin_scores(q, k, noise)
    # brute force: the two means summed element by element
    ref = np.zeros((B, Hkv, NQB, NQB))
    for b in range(B):
        for h in range(Hkv):
            for i in range(NQB):
                for j in range(NQB):
                    dot = 0.0
                    for d in range(D):
                        qm = sum(q[b, i * BLOCK + t, h * G + g, d] for t in range(BLOCK) for g in range(G)) / (BLOCK * G)
                        km = sum(k[b, j * BLOCK + t, h, d] for t in range(BLOCK)) / BLOCK
                        dot += qm * km
                    ref[b, h, i, j] = dot / math.sqrt(D) + noise[b, h, i, j]
    assert np.allclose(s, ref, rtol=1e-12, atol=1e-12)
    # closed form: constant q = a, k = c gives a * c * D / sqrt(D) = a * c * sqrt(D)
    sc = O.standin_scores(np.full((1, 128, 4, 16), 0.5), np.full((1, 128, 2, 16), -3.0), np.zeros((1, 2, 2, 2)))
    assert np.allclose(sc, 0.5 * -3.0 * math.sqrt(16), rtol=1e-14)
    # invariances: row order inside a block, and linearity in q
    perm = np.random.default_rng(34).permutation(BLOCK)
    qp = q.copy()
    qp[:, BLOCK:2 * BLOCK] = q[:, BLOCK + perm]
    assert np.allclose(O.standin_scores(qp, k, noise), s, rtol=1e-12, atol=1e-12)
    assert np.allclose(O.standin_scores(2.0 * q, k, noise) - noise, 2.0 * (s - noise), rtol=1e-12, atol=1e-12)
    # GQA map: query head hq pools into KV head hq // G only
    q1 = np.zeros_like(q)
    q1[:, :, G + 1, :] = q[:, :, G + 1, :]
    s1 = O.standin_scores(q1, k, np.zeros_like(noise))
    assert np.all(s1[:, 0] == 0.0) and np.any(s1[:, 1] != 0.0)


def _sas_bias(s_rows, L, K):
    """Additive mask of one sequence of L tokens (last block possibly partial) from
    the rank selection and scipy gates: [L, L]."""
    NQB = (L + BLOCK - 1) // BLOCK
    bias = np.full((L, L), -np.inf)
    for i in range(NQB):
        row = np.asarray(s_rows[i, :i], dtype=np.float64)
        ls = sp_logsumexp(row) if i else 0.0
        r0, r1 = i * BLOCK, min(L, (i + 1) * BLOCK)
        for j in _rank_select(list(row), K):
            bias[r0:r1, j * BLOCK:(j + 1) * BLOCK] = row[j] - ls
        for r in range(r0, r1):
            bias[r, r0:r + 1] = 0.0
    return bias


def pin_partial_block_sdpa(O):
    """A length that is not a multiple of 64: SDPA with the rank-selection mask."""
    S, Hq, Hkv, D, K = 229, 4, 2, 8, 2
    G = Hq // Hkv
    q, k, v = _rand((1, S, Hq, D), 121), _rand((1, S, Hkv, D), 122), _rand((1, S, Hkv, D), 123)
    NQB = 4
    s = _rand((1, Hkv, NQB, NQB), 124, 1.5).astype(np.float32)
    idx, cnt, lg, _ = O.select(s, K, O.prefill_history(NQB))
    sc = 1.0 / math.sqrt(D)
    o, lse = O.attn_fwd(q, k, v, idx, cnt, lg, sc)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    for h in range(Hkv):
        bias = _sas_bias(s[0, h], S, K)
        for g in range(G):
            hq = h * G + g
            ref = _sdpa(q[0, :, hq], k[0, :, h], v[0, :, h], bias, sc)
            assert np.allclose(o[0, :, hq], ref, rtol=1e-12, atol=1e-12)
            ref_lse = torch.logsumexp(torch.from_numpy(sc * q[0, :, hq] @ k[0, :, h].T + bias), dim=1).numpy()
            assert np.allclose(lse[0, hq], ref_lse, rtol=1e-12, atol=1e-12)


def pin_partial_block_prefix(O):
    """Causality: a sequence cut at S = 229 gives the first 229 rows of the same
    sequence at 256 (its last block full), forward and backward, when the longer
    sequence's extra rows carry no upstream gradient; the extra keys get none."""
    S, S2, Hq, Hkv, D, K = 229, 256, 4, 2, 8, 2
    q, k, v = _rand((1, S2, Hq, D), 131), _rand((1, S2, Hkv, D), 132), _rand((1, S2, Hkv, D), 133)
    do = _rand((1, S2, Hq, D), 134)
    do[:, S:] = 0.0
    s = _rand((1, Hkv, 4, 4), 135)
    sel = O.select(s, K, O.prefill_history(4))
    sc = 0.37
    o1, l1 = O.attn_fwd(q[:, :S], k[:, :S], v[:, :S], *sel[:3], sc)
    o2, l2 = O.attn_fwd(q, k, v, *sel[:3], sc)
    assert np.allclose(o1, o2[:, :S], rtol=0, atol=1e-13) and np.allclose(l1, l2[:, :, :S], rtol=0, atol=1e-13)
    g1 = O.attn_bwd(q[:, :S], k[:, :S], v[:, :S], do[:, :S], *sel[:3], s, sc)
    g2 = O.attn_bwd(q, k, v, do, *sel[:3], s, sc)
    for a, b in zip(g1[:3], g2[:3]):
        assert np.allclose(a, b[:, :S], rtol=0, atol=1e-12)
    assert np.all(g2[1][:, S:] == 0.0) and np.all(g2[2][:, S:] == 0.0)
    assert np.allclose(g1[3], g2[3], rtol=0, atol=1e-12)
    assert np.abs(g1[3]).max() > 1e-3       # the gate gradients are exercised


def _varlen_case(seed):
    lens = [100, 64, 1, 229, 0, 130]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T, Hq, Hkv, D = int(cu[-1]), 4, 2, 8
    q, k, v = _rand((T, Hq, D), seed), _rand((T, Hkv, D), seed + 1), _rand((T, Hkv, D), seed + 2)
    R = 4
    s = _rand((len(lens), Hkv, R, R), seed + 3).astype(np.float32)
    return lens, cu, q, k, v, s


def pin_varlen_sdpa(O):
    """A packed batch of sequences of lengths 100, 64, 1, 229, 0, 130 against SDPA over
    all packed rows with a mask that is each sequence's SAS mask on its diagonal block
    and -inf between sequences; padding rows of the selection are empty."""
    lens, cu, q, k, v, s = _varlen_case(141)
    K, Hq, Hkv, D = 2, 4, 2, 8
    G = Hq // Hkv
    T = int(cu[-1])
    idx, cnt, lg, lse_s = O.select_varlen(s, K, cu)
    for b, L in enumerate(lens):
        nb = (L + BLOCK - 1) // BLOCK
        assert np.all(cnt[b, :, nb:] == 0) and np.all(idx[b, :, nb:] == -1) and np.all(np.isneginf(lse_s[b, :, nb:]))
    sc = 1.0 / math.sqrt(D)
    o, lse = O.attn_fwd_varlen(q, k, v, cu, idx, cnt, lg, sc, max(lens))
    for h in range(Hkv):
        bias = np.full((T, T), -np.inf)
        for b, L in enumerate(lens):
            if L:
                st = int(cu[b])
                bias[st:st + L, st:st + L] = _sas_bias(s[b, h], L, K)
        for g in range(G):
            hq = h * G + g
            ref = _sdpa(q[:, hq], k[:, h], v[:, h], bias, sc)
            assert np.allclose(o[:, hq], ref, rtol=1e-12, atol=1e-12)
            ref_lse = torch.logsumexp(torch.from_numpy(sc * q[:, hq] @ k[:, h].T + bias), dim=1).numpy()
            for b, L in enumerate(lens):
                st = int(cu[b])
                assert np.allclose(lse[b, hq, :L], ref_lse[st:st + L], rtol=1e-12, atol=1e-12)
                assert np.all(np.isnan(lse[b, hq, L:]))


def pin_varlen_finite_differences(O):
    """Gradients of the packed batch against central finite differences of its loss."""
    lens, cu, q, k, v, s = _varlen_case(151)
    K, sc, h = 2, 0.3, 1e-6
    do = _rand(q.shape, 155)
    idx, cnt, lg, _ = O.select_varlen(s, K, cu)
    dq, dk, dv, ds = O.attn_bwd_varlen(q, k, v, do, cu, idx, cnt, lg, s, sc)

    def loss(q, k, v, s):
        sel = O.select_varlen(s, K, cu)
        o, _ = O.attn_fwd_varlen(q, k, v, cu, *sel[:3], sc, max(lens))
        return float(np.sum(o * do))

    r = np.random.default_rng(156)
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(8):
            pos = tuple(int(r.integers(0, n)) for n in grad.shape)
            args = dict(q=q, k=k, v=v)
            plus, minus = args[name].copy(), args[name].copy()
            plus[pos] += h
            minus[pos] -= h
            lp = loss(**{**args, name: plus}, s=s)
            lm = loss(**{**args, name: minus}, s=s)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])
    for b, i, j in ((0, 1, 0), (3, 3, 1), (3, 2, 0), (5, 2, 1)):
        plus, minus = s.copy(), s.copy()
        plus[b, 1, i, j] += np.float32(1e-3)
        minus[b, 1, i, j] -= np.float32(1e-3)
        step = float(plus[b, 1, i, j]) - float(minus[b, 1, i, j])
        fd = (loss(q, k, v, plus) - loss(q, k, v, minus)) / step
        assert abs(fd - ds[b, 1, i, j]) <= 1e-5 * max(1.0, abs(fd)), (b, i, j, fd, ds[b, 1, i, j])
    for b, L in enumerate(lens):
        nb = (L + BLOCK - 1) // BLOCK
        assert np.all(ds[b, :, nb:] == 0.0)


def pin_standin_scores_decode(O):
    """Decode stand-in scores against explicit loops, the prefill stand-in, a closed form
    and invariance to where the pages sit in the cache."""
    N, Hq, Hkv, D = 3, 6, 2, 8
    G = Hq // Hkv
    lens = [1, 130, 200]
    maxp = 4
    P = 12
    q = _rand((N, Hq, D), 161)
    kc = _rand((P, Hkv, BLOCK, D), 162)
    pt = np.array([[5, 0, 0, 0], [7, 2, 9, 0], [1, 11, 3, 4]])
    noise = _rand((N, Hkv, maxp), 163)
    s = O.standin_scores_decode(q, kc, pt, np.array(lens), noise)
    for n, L in enumerate(lens):
        nh = (L - 1) // BLOCK
        assert np.all(np.isnan(s[n, :, nh:]))
        for h in range(Hkv):
            for j in range(nh):
                dot = 0.0
                for d in range(D):
                    qm = sum(q[n, h * G + g, d] for g in range(G)) / G
                    km = sum(kc[pt[n, j], h, t, d] for t in range(BLOCK)) / BLOCK
                    dot += qm * km
                assert abs(s[n, h, j] - (dot / math.sqrt(D) + noise[n, h, j])) < 1e-12
    # a prefill query block whose 64 rows are one token repeated scores history blocks
    # like that token's decode query
    S = 3 * BLOCK
    kp = _rand((1, S, Hkv, D), 164)
    qp = np.repeat(q[2][None, None], BLOCK, axis=1)                   # [1, 64, Hq, D]
    qfull = np.concatenate([np.zeros((1, 2 * BLOCK, Hq, D)), qp], axis=1)
    sp = O.standin_scores(qfull, kp, np.zeros((1, Hkv, 3, 3)))
    kc2 = kp[0].reshape(3, BLOCK, Hkv, D).transpose(0, 2, 1, 3)       # pages 0, 1, 2 in order
    sd = O.standin_scores_decode(q[2:3], kc2, np.array([[0, 1, 2]]), np.array([2 * BLOCK + 1]),
                                 np.zeros((1, Hkv, 3)))
    assert np.allclose(sd[0, :, :2], sp[0, :, 2, :2], rtol=0, atol=1e-12)
    # closed form: constant q = a, k = c gives a * c * sqrt(D)
    c = O.standin_scores_decode(np.full((1, 4, 16), 0.5), np.full((2, 2, BLOCK, 16), -2.0), np.array([[1, 0]]),
                                np.array([129]), np.zeros((1, 2, 2)))
    assert np.allclose(c, 0.5 * -2.0 * 4.0, rtol=1e-14)
    # moving the pages elsewhere in the cache (and the table with them) changes nothing
    perm = np.random.default_rng(165).permutation(P)
    inv = np.argsort(perm)
    s2 = O.standin_scores_decode(q, kc[perm], inv[pt], np.array(lens), noise)
    assert np.array_equal(np.isnan(s), np.isnan(s2)) and np.allclose(s[~np.isnan(s)], s2[~np.isnan(s2)], rtol=0,
                                                                      atol=1e-13)


def pin_attended_tiles(O):
    """The attended-tile count the throughput is quoted on, by brute force: every
    query head of every query block attends its own block and each kept one."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, NQB, K = 2, 6, 2, 10, 3
    s = rng.standard_normal((B, Hkv, NQB, NQB))
    _, cnt, _, _ = O.select(s, K, O.prefill_history(NQB))
    brute = 0
    for b in range(B):
        for hq in range(Hq):
            for i in range(NQB):
                brute += 1 + min(K, i)          # own block + min(K, #history) kept ones
    assert O.attended_tiles(cnt, Hq, Hkv) == brute == B * Hq * (1 + 2 + 3 + 4 * 7)


ALL_PINS = [
    pin_topk_rank, pin_select_gates, pin_golden, pin_dense_equivalence, pin_block_diagonal,
    pin_general_sdpa, pin_bruteforce_loops, pin_finite_differences, pin_shift_invariance,
    pin_sparsity, pin_probabilities, pin_decode_vs_sdpa, pin_decode_vs_prefill, pin_standin_scores,
    pin_partial_block_sdpa, pin_partial_block_prefix, pin_varlen_sdpa, pin_varlen_finite_differences,
    pin_standin_scores_decode, pin_attended_tiles,
]
