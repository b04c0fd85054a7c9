"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Small cases: every output element, on sizes the oracle finishes in seconds
that still span several tiles, both GQA group sizes, both head dims, K = 0,
K >= #history and the fp32 path. Full workload sizes: select on every row,
and forward/backward/decode outputs on sampled stripes, key blocks and
sequences that the oracle computes one by one.
"""
import math
import random
import zlib

import numpy as np
import pytest
import torch

from oracle import sas_oracle as O
from tests.parity_util import check_grad, check_out, max_abs, np64
from trainable_gated_block_b200 import build, inputs, sas

pytestmark = pytest.mark.gpu
BLOCK = 64


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    sas.lib()


def _dev(d):
    return {k: v.cuda() for k, v in d.items()}


def _select_checks(s_cpu, K, gsel, n_hist, poison=True):
    idx, cnt, lg, lse_s = O.select(s_cpu, K, n_hist)
    gidx, gcnt, glg, glse = (t.cpu().numpy() for t in gsel)
    assert np.array_equal(gidx, idx), "Top-K indices differ"
    assert np.array_equal(gcnt, cnt), "counts differ"
    fin = np.isfinite(lg)
    assert np.array_equal(fin, np.isfinite(glg))
    assert np.all(np.isneginf(glg[~fin]))
    assert max_abs(glg[fin], lg[fin]) <= 1e-5
    finl = np.isfinite(lse_s)
    assert np.array_equal(finl, np.isfinite(glse))
    assert max_abs(glse[finl], lse_s[finl]) <= 1e-5
    return idx, cnt, lg, lse_s


def _poisoned(s):
    """NaN in every entry a row may not read (j >= i): proves they are never read."""
    s = s.clone()
    n = s.shape[-2]
    mask = torch.triu(torch.ones(n, s.shape[-1], dtype=torch.bool))
    s[..., mask] = float("nan")
    return s


# ---------------------------------------------------------------------------
# select
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny-fp32", "qwen3-4b-8k", "qwen3-8b-32k", "qwen3-14b-2x32k"])
def test_select_full_workloads(name):
    cfg = inputs.workload(name)
    g = torch.Generator().manual_seed(cfg.seed)
    B, H, NQB = cfg.B, cfg.Hkv, cfg.NQB
    # the scores only (same recipe shape; the standin scores are checked in the chain test)
    s = (torch.randn((B, H, NQB, NQB), generator=g) * cfg.score_std).float()
    sp = _poisoned(s)
    gsel = sas.select(sp.cuda(), cfg.K)
    torch.cuda.synchronize()
    sas.get_error_flag()
    _select_checks(s, cfg.K, gsel, O.prefill_history(NQB))


@pytest.mark.parametrize("R", [200, 700, 2000])   # one-warp rows; one-CTA rows (radix select) beyond 512
def test_select_adversarial_ties(R):
    rng = np.random.default_rng(5)
    B, H = 2, 3
    s = rng.choice(np.array([-1.0, -0.0, 0.0, 0.5, 2.0], dtype=np.float32), size=(B, H, R, R))
    s[0, 0] = 0.25                        # all-equal rows
    s[0, 1, :, ::2] = -0.0                # +/- zero ties
    s[0, 1, :, 1::2] = 0.0
    st = torch.from_numpy(s)
    for K in (0, 1, 7, 32, 199, 300, R + 5):
        gsel = sas.select(_poisoned(st).cuda(), K)
        sas.get_error_flag()
        _select_checks(st, K, gsel, O.prefill_history(R))


def test_select_decode_rows():
    cfg = inputs.workload("decode-64seq", partial=True)
    g = torch.Generator().manual_seed(77)
    N, H = cfg.N, cfg.Hkv
    kv_len = (torch.randint(1, 1024 * 64 + 1, (N,), generator=g)).to(torch.int32)
    kv_len[:6] = torch.tensor([1, 64, 65, 128, 129, 1024 * 64], dtype=torch.int32)
    s = torch.randn((N, H, 1024), generator=g)
    gsel = sas.select(s.cuda(), cfg.K, kv_len=kv_len.cuda())
    sas.get_error_flag()
    nh = O.decode_history(kv_len.numpy())
    _select_checks(s[:, :, None, :], cfg.K, [t[:, :, None] for t in gsel], nh[:, None])


# ---------------------------------------------------------------------------
# forward + backward, every element, small sizes
# ---------------------------------------------------------------------------

SMALL = [
    # name,       dtype, B, S,    Hq, Hkv, D,  K, score_std
    ("tiny-fp32", "f32", 1, 512, 2, 1, 64, 2, 1.0),
    ("f32-d128-g4", "f32", 1, 384, 4, 1, 128, 2, 1.0),
    ("bf16-g4", "bf16", 2, 1024, 8, 2, 128, 3, 1.0),
    ("bf16-g5", "bf16", 1, 768, 10, 2, 128, 4, 2.0),
    ("bf16-d64", "bf16", 1, 640, 4, 2, 64, 2, 1.0),
    ("bf16-K0", "bf16", 1, 512, 4, 1, 128, 0, 1.0),
    ("bf16-dense", "bf16", 1, 512, 4, 1, 128, 8, 1.0),
    ("bf16-one-block", "bf16", 2, 64, 8, 2, 128, 4, 1.0),
    # lengths that are not a multiple of 64 (a partial last block)
    ("bf16-S100-g4", "bf16", 2, 100, 8, 2, 128, 3, 1.0),
    ("f32-S229-d64", "f32", 1, 229, 2, 1, 64, 2, 1.0),
    ("bf16-S1000-g5", "bf16", 1, 1000, 10, 2, 128, 4, 2.0),
    ("bf16-S65-d64", "bf16", 1, 65, 4, 2, 64, 2, 1.0),
    ("bf16-S1", "bf16", 2, 1, 8, 2, 128, 2, 1.0),
    # other GQA group sizes on the tensor-core path: one head per KV head (a
    # padding head in every tile), two (one tile per group), three (one tile
    # and a half-padded one) and eight (two tiles in each of two groups)
    ("bf16-g1", "bf16", 1, 576, 2, 2, 128, 3, 1.0),
    ("bf16-g2", "bf16", 2, 448, 4, 2, 128, 2, 1.0),
    ("bf16-g3-S300", "bf16", 1, 300, 6, 2, 128, 2, 1.0),
    ("bf16-g8", "bf16", 1, 640, 8, 1, 128, 4, 1.0),
]


def _small_inputs(dtype, B, S, Hq, Hkv, D, K, std, seed):
    cfg = inputs.PrefillConfig("small", dtype, B, S, Hq, Hkv, D, K, "normal", std, seed=seed)
    return cfg, inputs.make_prefill(cfg)


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_fwd_bwd_small(case):
    name, dtype, B, S, Hq, Hkv, D, K, std = case
    cfg, x = _small_inputs(dtype, B, S, Hq, Hkv, D, K, std, seed=zlib.crc32(name.encode()) % 1000)
    NQB = cfg.NQB
    sc = 1.0 / math.sqrt(D)
    xd = _dev(x)
    gsel = sas.select(_poisoned(x["s"]).cuda(), K)
    idx, cnt, lg, lse_s = _select_checks(x["s"], K, gsel, O.prefill_history(NQB))
    o, lse = sas.attn_fwd(xd["q"], xd["k"], xd["v"], gsel[0], gsel[1], gsel[2], sc)
    dq, dk, dv, ds = sas.attn_bwd(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, xd["s"], gsel[3],
                                  gsel[0], gsel[1], gsel[2], sc)
    torch.cuda.synchronize()
    sas.get_error_flag()
    ro, rlse = O.attn_fwd(x["q"], x["k"], x["v"], idx, cnt, lg, sc)
    rdq, rdk, rdv, rds, _ = O.attn_bwd(x["q"], x["k"], x["v"], x["do"], idx, cnt, lg, x["s"], sc)
    check_out(o, ro, dtype, "o")
    check_out(lse, rlse, "f32" if dtype == "f32" else dtype, "lse")
    check_grad(dq, rdq, dtype, "dq")
    check_grad(dk, rdk, dtype, "dk")
    check_grad(dv, rdv, dtype, "dv")
    check_grad(ds, rds, dtype, "ds")
    # rows of ds sum to zero (shift invariance of the gates in s)
    dsn = np64(ds)
    assert np.all(np.abs(dsn.sum(-1)) <= 1e-4 * (1 + np.abs(dsn).sum(-1)))


def test_unselected_kv_has_no_influence_on_gpu():
    cfg, x = _small_inputs("bf16", 1, 1024, 8, 2, 128, 2, 1.0, seed=9)
    xd = _dev(x)
    sel = sas.select(xd["s"], 2)
    o1, l1 = sas.attn_fwd(xd["q"], xd["k"], xd["v"], *sel[:3])
    idx = sel[0].cpu().numpy()
    cnt = sel[1].cpu().numpy()
    i = 15
    keep = {int(j) for h in range(2) for j in idx[0, h, i, :cnt[0, h, i]]} | {i}
    k2, v2 = x["k"].clone(), x["v"].clone()
    for j in range(16):
        if j not in keep:
            k2[0, j * 64:(j + 1) * 64] = torch.randn(64, 2, 128).bfloat16() * 3
            v2[0, j * 64:(j + 1) * 64] = torch.randn(64, 2, 128).bfloat16() * 3
    o2, l2 = sas.attn_fwd(xd["q"], k2.cuda(), v2.cuda(), *sel[:3])
    rs = slice(i * 64, (i + 1) * 64)
    assert torch.equal(o1[0, rs], o2[0, rs]) and torch.equal(l1[0, :, rs], l2[0, :, rs])


def test_bad_indices_are_flagged_not_followed():
    cfg, x = _small_inputs("bf16", 1, 256, 4, 1, 128, 2, 1.0, seed=3)
    xd = _dev(x)
    idx, cnt, lg, _ = sas.select(xd["s"], 2)
    idx = idx.clone()
    idx[0, 0, 3, 0] = 7              # not a history block of query block 3
    sas.get_error_flag()
    o, _ = sas.attn_fwd(xd["q"], xd["k"], xd["v"], idx, cnt, lg)
    with pytest.raises(sas.SasError) as e:
        sas.get_error_flag()
    assert e.value.code == sas.SAS_ERR_INVALID_ARG
    sas.get_error_flag()             # cleared


def test_bounded_wait_timeout_is_reported_and_context_survives():
    """Failure detection without a GPU fault: a wait that can never complete gives up on
    its budget, the host reads SAS_ERR_TIMEOUT once, and the next call runs normally."""
    sas.get_error_flag()                 # nothing pending
    sas.selftest_bounded_wait()
    with pytest.raises(sas.SasError) as e:
        sas.get_error_flag()
    assert e.value.code == sas.SAS_ERR_TIMEOUT
    sas.get_error_flag()                 # reported once, then cleared
    s = torch.from_numpy(np.random.default_rng(11).standard_normal((1, 2, 40, 40)).astype(np.float32))
    gsel = sas.select(_poisoned(s).cuda(), 5)
    sas.get_error_flag()
    _select_checks(s, 5, gsel, O.prefill_history(40))


# ---------------------------------------------------------------------------
# full workload sizes, sampled
# ---------------------------------------------------------------------------

def _reverse(idx, cnt, b, h, j):
    """Query blocks that attend key block j (its own block and every selector)."""
    rows = [j]
    NQB = idx.shape[2]
    for i in range(j + 1, NQB):
        if j in idx[b, h, i, :cnt[b, h, i]]:
            rows.append(i)
    return rows


@pytest.mark.parametrize("name", ["qwen3-4b-8k", "qwen3-8b-32k", "qwen3-14b-2x32k"])
def test_full_workload_sampled(name):
    cfg = inputs.workload(name)
    NQB = cfg.NQB
    rnd = random.Random(cfg.seed)
    _sampled_parity(cfg, [0, 1, NQB // 2, NQB - 1, rnd.randrange(NQB)])


def test_mixed_tile_items_sampled():
    """GQA group of 10: head groups of 4, 4 and 2 heads, so the forward's items alternate
    between two Q tiles and one on the same CTA (384 items over a 148-CTA grid). Query blocks
    0, 1, 15 and 64 are processed after an item with an idle tile on their CTA; 100 and 127
    are first items."""
    cfg = inputs.PrefillConfig("g10-mixed", "bf16", 1, 8192, 10, 1, 128, 8, "normal", 1.0, seed=21)
    _sampled_parity(cfg, [0, 1, 15, 64, 100, 127])


def _dkv_picks(idx, cnt, b, h, G, NQB, rnd, budget, extra=()):
    """Key blocks whose dk/dv the oracle recomputes: the last two, the block kept by the
    most query blocks (the most kept one whose attending stripes fit the budget), blocks
    given in ``extra``, and one attended by a handful of query blocks."""
    picks = [NQB - 1, max(NQB - 2, 0)] + [j for j in extra if 0 <= j < NQB]
    kept = np.bincount(idx[b, h][idx[b, h] >= 0].ravel(), minlength=NQB)
    for j in np.argsort(-kept, kind="stable"):
        if (kept[j] + 1) * G <= budget:
            picks.append(int(j))
            break
    for j in rnd.sample(range(NQB), min(NQB, 40)):
        if 3 <= len(_reverse(idx, cnt, b, h, j)) <= 12 and j not in picks:
            picks.append(j)
            break
    return list(dict.fromkeys(picks))


def _sampled_parity(cfg, rows, heads=2, dkv_extra=(), dkv_budget=800):
    """Full-size run on the GPU; the oracle recomputes sampled stripes one by one: o, lse
    and dq of the given query blocks (all heads of the sampled KV heads), their ds rows, and
    dk/dv of at least four key blocks per sampled KV head."""
    x = inputs.make_prefill(cfg)
    xd = _dev(x)
    NQB, G, D, S = cfg.NQB, cfg.G, cfg.D, cfg.S
    sc = 1.0 / math.sqrt(D)
    gsel = sas.select(xd["s"], cfg.K)
    o, lse = sas.attn_fwd(xd["q"], xd["k"], xd["v"], *gsel[:3], sc)
    dq, dk, dv, ds = sas.attn_bwd(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, xd["s"], gsel[3],
                                  gsel[0], gsel[1], gsel[2], sc)
    torch.cuda.synchronize()
    sas.get_error_flag()
    idx, cnt, lg, _ = _select_checks(x["s"], cfg.K, gsel, O.prefill_history(NQB))
    rnd = random.Random(cfg.seed + 1)
    b = cfg.B - 1
    for h in rnd.sample(range(cfg.Hkv), min(heads, cfg.Hkv)):
        stripes = [(b, h * G + g, i) for i in rows for g in range(G)]
        ro, rlse = O.attn_fwd(x["q"], x["k"], x["v"], idx, cnt, lg, sc, stripes=stripes)
        rdq, _, _, rds, _ = O.attn_bwd(x["q"], x["k"], x["v"], x["do"], idx, cnt, lg, x["s"], sc, stripes=stripes)
        for (bb, hq, i) in stripes:
            rs = O.block_rows(i, S)
            check_out(o[bb, rs, hq], ro[bb, rs, hq], "bf16", f"{cfg.name} o[{bb},{i},{hq}]")
            check_out(lse[bb, hq, rs], rlse[bb, hq, rs], "bf16", f"{cfg.name} lse[{bb},{i},{hq}]")
        dq_s = np.concatenate([np64(dq[bb, O.block_rows(i, S), hq]) for bb, hq, i in stripes])
        rdq_s = np.concatenate([rdq[bb, O.block_rows(i, S), hq] for bb, hq, i in stripes])
        check_grad(dq_s, rdq_s, "bf16", f"{cfg.name} dq (sampled stripes, KV head {h})")
        ds_s = np.stack([np64(ds[b, h, i, :NQB]) for i in rows])
        rds_s = np.stack([rds[b, h, i, :NQB] for i in rows])
        check_grad(ds_s, rds_s, "bf16", f"{cfg.name} ds (sampled rows, KV head {h})")
        picks = _dkv_picks(idx, cnt, b, h, G, NQB, rnd, dkv_budget, dkv_extra)
        assert len(picks) >= 4 or NQB < 4
        for j in picks:
            att = _reverse(idx, cnt, b, h, j)
            kst = [(b, h * G + g, i) for i in att for g in range(G)]
            _, rdk, rdv, _, _ = O.attn_bwd(x["q"], x["k"], x["v"], x["do"], idx, cnt, lg, x["s"], sc, stripes=kst)
            ks = O.block_rows(j, S)
            check_grad(dk[b, ks, h], rdk[b, ks, h], "bf16", f"{cfg.name} dk block {j} (KV head {h}, {len(att)} rows)")
            check_grad(dv[b, ks, h], rdv[b, ks, h], "bf16", f"{cfg.name} dv block {j} (KV head {h}, {len(att)} rows)")
    return idx, cnt


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def _decode_run(x, K):
    xd = _dev(x)
    sel = sas.select(xd["s"], K, kv_len=xd["kv_len"])
    o, lse = sas.decode_paged(xd["q"], xd["k_cache"], xd["v_cache"], xd["page_table"], xd["kv_len"],
                              sel[0], sel[1], sel[2])
    torch.cuda.synchronize()
    sas.get_error_flag()
    return sel, o, lse


def _decode_oracle_check(x, K, sel, o, lse, seqs):
    s4 = x["s"][:, :, None, :]
    idx, cnt, lg, _ = _select_checks(s4, K, [t[:, :, None] for t in sel], O.decode_history(x["kv_len"])[:, None])
    ro, rlse = O.decode(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["kv_len"],
                        idx[:, :, 0], cnt[:, :, 0], lg[:, :, 0], 1.0 / math.sqrt(x["q"].shape[-1]), seqs=seqs)
    for n in seqs:
        check_out(o[n], ro[n], "bf16", f"decode o[{n}]")
        check_out(lse[n], rlse[n], "bf16", f"decode lse[{n}]")


@pytest.mark.parametrize("G,partial", [(4, True), (4, False), (5, True), (1, True), (8, True)])
def test_decode_small(G, partial):
    cfg = inputs.DecodeConfig("small", N=6, Hq=2 * G, Hkv=2, D=128, K=5, min_hist=0, max_hist=24,
                              partial=partial, seed=10 + G)
    x = inputs.make_decode(cfg)
    x["kv_len"][0] = 1
    x["kv_len"][1] = min(int(x["kv_len"][1]), 64)
    sel, o, lse = _decode_run(x, cfg.K)
    _decode_oracle_check(x, cfg.K, sel, o, lse, range(cfg.N))


def test_decode_full_workload_sampled():
    cfg = inputs.workload("decode-64seq")
    x = inputs.make_decode(cfg)
    sel, o, lse = _decode_run(x, cfg.K)
    longest = int(torch.argmax(x["kv_len"]))
    shortest = int(torch.argmin(x["kv_len"]))
    _decode_oracle_check(x, cfg.K, sel, o, lse, sorted({0, 31, 63, longest, shortest}))
