"""Parity through the C ABI of the paths beyond the dense, block-aligned case:
sequence lengths that end in a partial block, packed batches of sequences of
different lengths, the full-history variant (K >= #history) at full size,
select on long decode rows (the CTA radix select) and select on rows that hold
non-finite scores.
"""
import math
import random

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import sas_oracle as O
from tests.parity_util import check_grad, check_out, max_abs, np64
from tests.test_gpu_parity import _dev, _poisoned, _reverse, _sampled_parity, _select_checks
from trainable_gated_block_b200 import build, inputs, sas

pytestmark = pytest.mark.gpu
BLOCK = 64


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    sas.lib()


# ---------------------------------------------------------------------------
# select: rows with non-finite scores, long decode rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("R", [40, 700])            # warp-per-row and CTA-per-row kernels
def test_select_nonfinite_rows_are_flagged(R):
    rng = np.random.default_rng(R)
    s = rng.standard_normal((2, 2, R, R)).astype(np.float32)
    bad = {(0, 0, 5): np.nan, (0, 1, 17): np.inf, (1, 0, 30): -np.inf, (1, 1, R - 1): np.nan}
    for (b, h, i), val in bad.items():
        s[b, h, i, i // 2] = val                   # inside the row's history
    s[0, 0, 3, 3:] = np.nan                         # outside it: never read
    sas.get_error_flag()
    gsel = sas.select(torch.from_numpy(s).cuda(), 4)
    with pytest.raises(sas.SasError) as e:
        sas.get_error_flag()
    assert e.value.code == sas.SAS_ERR_INVALID_ARG
    gidx, gcnt, glg, glse = (t.cpu().numpy() for t in gsel)
    ok = np.ones((2, 2, R), dtype=bool)
    s_ok = s.copy()
    for (b, h, i) in bad:
        ok[b, h, i] = False
        assert gcnt[b, h, i] == 0 and np.all(gidx[b, h, i] == -1)
        assert np.all(np.isneginf(glg[b, h, i])) and np.isnan(glse[b, h, i])
        with pytest.raises(ValueError):            # the oracle defines no Top-K for such a row
            O.topk_history(s[b, h, i], i, 4)
        s_ok[b, h, i] = 0.0
    idx, cnt, lg, lse_s = O.select(s_ok, 4, O.prefill_history(R))
    assert np.array_equal(gidx[ok], idx[ok]) and np.array_equal(gcnt[ok], cnt[ok])
    fin = np.isfinite(lg[ok])
    assert np.array_equal(fin, np.isfinite(glg[ok])) and max_abs(glg[ok][fin], lg[ok][fin]) <= 1e-5
    finl = np.isfinite(lse_s[ok])
    assert max_abs(glse[ok][finl], lse_s[ok][finl]) <= 1e-5


@pytest.mark.parametrize("max_blocks,K", [(4096, 32), (8192, 16), (16384, 32), (16384, 3000)])
def test_select_long_decode_rows(max_blocks, K):
    """Decode rows of up to 16384 history blocks (1M tokens): bit-exact Top-K, with tie-heavy
    and all-equal rows among them."""
    g = torch.Generator().manual_seed(max_blocks + K)
    N, H = 6, 8
    kv_len = torch.randint(1, max_blocks * 64 + 2, (N,), generator=g).to(torch.int32)
    kv_len[:3] = torch.tensor([1, max_blocks * 64 + 1, 64 * (max_blocks // 2) + 5], dtype=torch.int32)
    s = torch.randn((N, H, max_blocks), generator=g)
    s[3] = torch.round(s[3] * 2) / 2                # many ties
    s[4] = 0.25                                     # all equal
    gsel = sas.select(s.cuda(), K, kv_len=kv_len.cuda())
    sas.get_error_flag()
    nh = O.decode_history(kv_len.numpy())
    _select_checks(s[:, :, None, :], K, [t[:, :, None] for t in gsel], nh[:, None])


# ---------------------------------------------------------------------------
# partial last blocks at full size
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("S", [4095, 8193])
def test_partial_block_sampled(S):
    """Qwen3-4B-shaped heads (32/8, D=128, K=16) at lengths that end in a partial block:
    the partial block's rows, its keys' dk/dv, and blocks across the sequence."""
    cfg = inputs.PrefillConfig(f"partial-{S}", "bf16", 1, S, 32, 8, 128, 16, "normal", 1.0, seed=S)
    NQB = cfg.NQB
    _sampled_parity(cfg, [0, 1, NQB // 2, NQB - 2, NQB - 1], dkv_extra=(NQB - 1,))


# ---------------------------------------------------------------------------
# packed batches of sequences of different lengths
# ---------------------------------------------------------------------------

VARLEN = [
    # name, lengths, dtype, Hq, Hkv, D, K
    ("bf16-3seq", [100, 777, 1], "bf16", 8, 2, 128, 3),
    ("bf16-5seq-empty", [64, 0, 300, 129, 65], "bf16", 10, 2, 128, 2),
    ("f32-3seq-d64", [70, 190, 33], "f32", 4, 2, 64, 2),
]


def _varlen_run(x, K):
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    D = x["q"].shape[-1]
    sc = 1.0 / math.sqrt(D)
    gsel = sas.select_varlen(_poisoned(x["s"]).cuda(), K, xd["cu_seqlens"])
    o, lse = sas.attn_fwd_varlen(xd["q"], xd["k"], xd["v"], xd["cu_seqlens"], x["max_seqlen"], *gsel[:3], sc)
    # the selection also goes to the backward with scores whose unread entries are NaN
    sp = _poisoned(x["s"]).cuda()
    grads = sas.attn_bwd_varlen(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, sp, gsel[3], *gsel[:3],
                                xd["cu_seqlens"], x["max_seqlen"], sc)
    torch.cuda.synchronize()
    sas.get_error_flag()
    return gsel, o, lse, grads, sc


def _varlen_select_checks(x, K, gsel):
    idx, cnt, lg, lse_s = O.select_varlen(x["s"], K, x["cu_seqlens"])
    gidx, gcnt, glg, glse = (t.cpu().numpy() for t in gsel)
    assert np.array_equal(gidx, idx) and np.array_equal(gcnt, cnt)
    fin = np.isfinite(lg)
    assert np.array_equal(fin, np.isfinite(glg)) and max_abs(glg[fin], lg[fin]) <= 1e-5
    finl = np.isfinite(lse_s)
    assert np.array_equal(finl, np.isfinite(glse)) and max_abs(glse[finl], lse_s[finl]) <= 1e-5
    return idx, cnt, lg


@pytest.mark.parametrize("case", VARLEN, ids=[c[0] for c in VARLEN])
def test_varlen_every_element(case):
    name, lengths, dtype, Hq, Hkv, D, K = case
    x = inputs.make_varlen(lengths, Hq, Hkv, D, dtype, seed=len(name))
    gsel, o, lse, (dq, dk, dv, ds), sc = _varlen_run(x, K)
    idx, cnt, lg = _varlen_select_checks(x, K, gsel)
    ro, rlse = O.attn_fwd_varlen(x["q"], x["k"], x["v"], x["cu_seqlens"], idx, cnt, lg, sc, x["max_seqlen"])
    rdq, rdk, rdv, rds = O.attn_bwd_varlen(x["q"], x["k"], x["v"], x["do"], x["cu_seqlens"], idx, cnt, lg,
                                          x["s"], sc)
    check_out(o, ro, dtype, f"{name} o")
    for b, L in enumerate(lengths):
        check_out(lse[b, :, :L], rlse[b, :, :L], dtype, f"{name} lse seq {b}")
    check_grad(dq, rdq, dtype, f"{name} dq")
    check_grad(dk, rdk, dtype, f"{name} dk")
    check_grad(dv, rdv, dtype, f"{name} dv")
    check_grad(ds, rds, dtype, f"{name} ds")


def test_varlen_matches_dense_per_sequence():
    """Each sequence of a packed batch gives the same bits as the dense entry points run
    on that sequence alone (same kernels, so the same rounding); ds only to within the
    fp32 rounding of its atomically summed gate gradients."""
    lengths = [333, 64, 1000]
    x = inputs.make_varlen(lengths, 8, 2, 128, "bf16", seed=5)
    gsel, o, lse, (dq, dk, dv, ds), sc = _varlen_run(x, 4)
    cu = x["cu_seqlens"].tolist()
    for b, L in enumerate(lengths):
        rows = slice(cu[b], cu[b + 1])
        nb = (L + 63) // 64
        q1, k1, v1, do1 = (x[n][rows][None].cuda().contiguous() for n in ("q", "k", "v", "do"))
        s1 = _poisoned(x["s"][b:b + 1, :, :nb, :nb]).cuda().contiguous()
        sel1 = sas.select(s1, 4)
        o1, l1 = sas.attn_fwd(q1, k1, v1, *sel1[:3], sc)
        g1 = sas.attn_bwd(q1, k1, v1, o1, do1, l1, s1, sel1[3], *sel1[:3], sc)
        torch.cuda.synchronize()
        sas.get_error_flag()
        assert torch.equal(o[rows], o1[0]) and torch.equal(lse[b, :, :L], l1[0])
        assert torch.equal(dq[rows], g1[0][0]) and torch.equal(dk[rows], g1[1][0]) and torch.equal(dv[rows], g1[2][0])
        assert torch.allclose(ds[b, :, :nb, :nb], g1[3][0], rtol=1e-5, atol=1e-6)
        assert torch.all(ds[b, :, nb:] == 0)


def test_varlen_large_sampled():
    """A ragged batch of 4095, 8193, 64 and 1000 tokens, Qwen3-4B heads: sampled stripes of
    every sequence (including each partial last block) and dk/dv of key blocks of the
    longest sequence."""
    lengths = [4095, 8193, 64, 1000]
    Hq, Hkv, D, K = 32, 8, 128, 16
    G = Hq // Hkv
    x = inputs.make_varlen(lengths, Hq, Hkv, D, "bf16", seed=77)
    gsel, o, lse, (dq, dk, dv, ds), sc = _varlen_run(x, K)
    idx, cnt, lg = _varlen_select_checks(x, K, gsel)
    cu = x["cu_seqlens"].tolist()
    rnd = random.Random(78)
    for b, L in enumerate(lengths):
        nb = (L + 63) // 64
        rows = slice(cu[b], cu[b + 1])
        xs = {n: x[n][rows][None] for n in ("q", "k", "v", "do")}
        sb = x["s"][b:b + 1, :, :nb, :nb]
        ib, cb, lb = idx[b:b + 1, :, :nb], cnt[b:b + 1, :, :nb], lg[b:b + 1, :, :nb]
        h = rnd.randrange(Hkv)
        blocks = sorted({0, nb // 2, nb - 1})
        stripes = [(0, h * G + g, i) for i in blocks for g in range(G)]
        ro, rlse = O.attn_fwd(xs["q"], xs["k"], xs["v"], ib, cb, lb, sc, stripes=stripes)
        rdq, _, _, rds, _ = O.attn_bwd(xs["q"], xs["k"], xs["v"], xs["do"], ib, cb, lb, sb, sc, stripes=stripes)
        for (_, hq, i) in stripes:
            rs = O.block_rows(i, L)
            check_out(o[rows][rs, hq], ro[0, rs, hq], "bf16", f"varlen seq {b} o[{i},{hq}]")
            check_out(lse[b, hq, rs], rlse[0, hq, rs], "bf16", f"varlen seq {b} lse[{i},{hq}]")
        dq_s = np.concatenate([np64(dq[rows][O.block_rows(i, L), hq]) for _, hq, i in stripes])
        rdq_s = np.concatenate([rdq[0, O.block_rows(i, L), hq] for _, hq, i in stripes])
        check_grad(dq_s, rdq_s, "bf16", f"varlen seq {b} dq")
        check_grad(np.stack([np64(ds[b, h, i, :nb]) for i in blocks]), np.stack([rds[0, h, i] for i in blocks]),
                   "bf16", f"varlen seq {b} ds")
        if L == max(lengths):
            for j in (nb - 1, nb - 2, 1):
                att = _reverse(ib, cb, 0, h, j)
                kst = [(0, h * G + g, i) for i in att for g in range(G)]
                _, rdk, rdv, _, _ = O.attn_bwd(xs["q"], xs["k"], xs["v"], xs["do"], ib, cb, lb, sb, sc, stripes=kst)
                ks = O.block_rows(j, L)
                check_grad(dk[rows][ks, h], rdk[0, ks, h], "bf16", f"varlen seq {b} dk block {j}")
                check_grad(dv[rows][ks, h], rdv[0, ks, h], "bf16", f"varlen seq {b} dv block {j}")


def test_varlen_bad_bounds_are_flagged():
    """A sequence longer than max_seqlen is flagged and treated as empty; the others run."""
    lengths = [100, 200]
    x = inputs.make_varlen(lengths, 4, 2, 128, "bf16", seed=9)
    xd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    sel = sas.select_varlen(xd["s"], 2, xd["cu_seqlens"])
    sas.get_error_flag()
    sel3 = [t[:, :, :3].contiguous() for t in sel[:3]]     # blocks of a 150-token sequence
    o, lse = sas.attn_fwd_varlen(xd["q"], xd["k"], xd["v"], xd["cu_seqlens"], 150, *sel3)
    with pytest.raises(sas.SasError) as e:
        sas.get_error_flag()
    assert e.value.code == sas.SAS_ERR_INVALID_ARG
    o_ok, _ = sas.attn_fwd_varlen(xd["q"], xd["k"], xd["v"], xd["cu_seqlens"], 200, *sel[:3])
    sas.get_error_flag()
    assert torch.equal(o[:100], o_ok[:100])


# ---------------------------------------------------------------------------
# the full-history variant (K >= #history) at full size
# ---------------------------------------------------------------------------

def test_full_history_8k_sampled():
    """Qwen3-4B layer at 8k with K = 128 >= every row's history: every query block keeps
    all its history, so key block 0 is attended by all 128 query blocks."""
    cfg = inputs.workload("qwen3-4b-8k", K=128)
    NQB = cfg.NQB
    idx, cnt = _sampled_parity(cfg, [0, 1, 64, NQB - 1], heads=1, dkv_extra=(0, 1), dkv_budget=600)
    assert np.array_equal(cnt[0, 0], np.arange(NQB))


def test_full_history_uniform_scores_is_dense_8k():
    """K >= #history and equal scores give dense causal attention with every history logit
    shifted by -ln(i) (query block i): checked against torch's fp64 attention with that
    additive mask on sampled query blocks, with no oracle involved."""
    cfg = inputs.workload("qwen3-4b-8k", K=128)
    x = inputs.make_prefill(cfg, with_do=False)
    S, G, D, NQB = cfg.S, cfg.G, cfg.D, cfg.NQB
    s = torch.zeros((1, cfg.Hkv, NQB, NQB))
    xd = _dev(dict(q=x["q"], k=x["k"], v=x["v"], s=s))
    sc = 1.0 / math.sqrt(D)
    sel = sas.select(xd["s"], cfg.K)
    o, lse = sas.attn_fwd(xd["q"], xd["k"], xd["v"], *sel[:3], sc)
    torch.cuda.synchronize()
    sas.get_error_flag()
    for i in (1, 2, 77, NQB - 1):
        rows = slice(i * 64, (i + 1) * 64)
        keys = (i + 1) * 64
        t = torch.arange(i * 64, (i + 1) * 64)[:, None]
        u = torch.arange(keys)[None, :]
        bias = torch.where(u < i * 64, torch.tensor(-math.log(i), dtype=torch.float64),
                           torch.where(u <= t, torch.tensor(0.0, dtype=torch.float64),
                                       torch.tensor(-math.inf, dtype=torch.float64)))
        for hq in (0, G + 1, cfg.Hq - 1):
            h = hq // G
            qr = x["q"][0, rows, hq].double()[None, None]
            kr = x["k"][0, :keys, h].double()[None, None]
            vr = x["v"][0, :keys, h].double()[None, None]
            ref = F.scaled_dot_product_attention(qr, kr, vr, attn_mask=bias[None, None], scale=sc)[0, 0]
            check_out(o[0, rows, hq], ref.numpy(), "bf16", f"dense-equivalence o[{i},{hq}]")
            ref_lse = torch.logsumexp(sc * qr[0, 0] @ kr[0, 0].T + bias, dim=1)
            check_out(lse[0, hq, rows], ref_lse.numpy(), "bf16", f"dense-equivalence lse[{i},{hq}]")


# ---------------------------------------------------------------------------
# decode at long context
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("K", [32, 4096])
def test_decode_256k_context(K):
    """Paged decode at 256K tokens of context (4096 history blocks per sequence, the
    CTA-per-row radix select), sparse (K = 32) and keeping every history block."""
    from tests.test_gpu_parity import _decode_oracle_check, _decode_run
    cfg = inputs.DecodeConfig("decode-256k", N=2, Hq=8, Hkv=2, D=128, K=K, min_hist=4095, max_hist=4096,
                              partial=True, seed=256)
    x = inputs.make_decode(cfg)                     # 4095-4096 history blocks + 1..64 tokens
    sel, o, lse = _decode_run(x, cfg.K)
    _decode_oracle_check(x, cfg.K, sel, o, lse, [0, 1])
