"""The stand-in scorer + select (sas_score_select) through the C ABI against the
oracle's fp64 stand-in scores (oracle.standin_scores) and Top-K (oracle.select).

The GPU sums the bf16 inputs in fp32, so its scores differ from the fp64 oracle's by
rounding: they must agree within SCORE_TOL. The selection is then compared with the
oracle's selection on the oracle's scores: bit-exact on every row whose K-th and
(K+1)-th largest scores are more than 2 * SCORE_TOL apart (rounding cannot reorder
them), and on the other rows it must be a valid Top-K within that bound.
"""
import math

import numpy as np
import pytest
import torch

from oracle import sas_oracle as O
from tests.parity_util import max_abs
from trainable_gated_block_b200 import build, inputs, sas

pytestmark = pytest.mark.gpu
SCORE_TOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    sas.lib()


def _check_head(x, sel, s_gpu, h, G, K, name):
    NQB = s_gpu.shape[-1]
    q, k, noise = x["q"], x["k"], x.get("noise")
    nz = noise[:, h:h + 1] if noise is not None else torch.zeros((q.shape[0], 1, NQB, NQB))
    s_ref = O.standin_scores(q[:, :, h * G:(h + 1) * G], k[:, :, h:h + 1], nz)     # [B, 1, NQB, NQB]
    tril = np.tril(np.ones((NQB, NQB), dtype=bool), -1)
    sg = s_gpu[:, h:h + 1].cpu().numpy().astype(np.float64)
    err = np.abs(sg - s_ref)[..., tril]
    assert err.max() <= SCORE_TOL, f"{name}: scores differ by {err.max():.3e}"
    ridx, rcnt, rlg, rlse = O.select(s_ref, K, O.prefill_history(NQB))
    gidx, gcnt, glg, glse = (t[:, h:h + 1].cpu().numpy() for t in sel)
    assert np.array_equal(gcnt, rcnt)
    fin = np.isfinite(rlse)
    assert max_abs(glse[fin], rlse[fin]) <= SCORE_TOL
    close = 0
    for b in range(s_ref.shape[0]):
        for i in range(NQB):
            c = int(rcnt[b, 0, i])
            row = s_ref[b, 0, i, :i]
            if c == i:                               # every history block kept
                assert list(gidx[b, 0, i, :c]) == list(range(i))
            else:
                srt = np.sort(row)[::-1]
                if srt[c - 1] - srt[c] > 2 * SCORE_TOL:
                    assert np.array_equal(gidx[b, 0, i], ridx[b, 0, i]), (name, b, i)
                else:                                # a near tie at the boundary
                    close += 1
                    g = gidx[b, 0, i, :c]
                    assert np.all(np.diff(g) > 0) and np.all(g >= 0) and np.all(g < i)
                    assert np.all(row[g] >= srt[c - 1] - 2 * SCORE_TOL)
            assert np.all(gidx[b, 0, i, c:] == -1)
            if c:
                exp = sg[b, 0, i, gidx[b, 0, i, :c]] - float(glse[b, 0, i])
                ref = row[gidx[b, 0, i, :c]] - float(rlse[b, 0, i])
                assert np.max(np.abs(glg[b, 0, i, :c] - ref)) <= 2 * SCORE_TOL
                assert np.max(np.abs(glg[b, 0, i, :c] - exp)) <= 1e-5
    return close


@pytest.mark.parametrize("name,h_list", [("standin-small", (0, 1)), ("qwen3-4b-8k", (0, 5)),
                                         ("qwen3-8b-32k", (3,))])
def test_score_select_against_oracle(name, h_list):
    if name == "standin-small":
        cfg = inputs.PrefillConfig(name, "bf16", 2, 1024, 10, 2, 128, 3, "standin", seed=12)
    else:
        cfg = inputs.workload(name)
    x = inputs.make_prefill(cfg, with_do=False)
    qd, kd, nd = x["q"].cuda(), x["k"].cuda(), x["noise"].cuda()
    s_gpu, *sel = sas.score_select(qd, kd, cfg.K, noise=nd)
    torch.cuda.synchronize()
    sas.get_error_flag()
    for h in h_list:
        _check_head(x, sel, s_gpu, h, cfg.G, cfg.K, name)


def test_score_select_without_noise_and_long_rows():
    """No noise (the pooled dot product alone), and rows of more than 512 history blocks
    (scores written first, then the CTA-per-row selection)."""
    cfg = inputs.PrefillConfig("standin-long", "bf16", 1, 40000 // 64 * 64, 4, 1, 64, 5, "standin", seed=13)
    x = inputs.make_prefill(cfg, with_do=False)
    x.pop("noise")
    s_gpu, *sel = sas.score_select(x["q"].cuda(), x["k"].cuda(), cfg.K)
    torch.cuda.synchronize()
    sas.get_error_flag()
    _check_head(x, sel, s_gpu, 0, cfg.G, cfg.K, "standin-long")


def test_score_select_feeds_the_backward():
    """The scores sas_score_select writes are the ones the backward's Jacobian reads: a full
    select -> forward -> backward chain from them matches the chain from sas_select on the
    same scores."""
    cfg = inputs.PrefillConfig("standin-chain", "bf16", 1, 2048, 8, 2, 128, 4, "standin", seed=14)
    x = inputs.make_prefill(cfg)
    xd = {k: v.cuda() for k, v in x.items()}
    sc = 1.0 / math.sqrt(cfg.D)
    s_gpu, idx, cnt, lg, lse_s = sas.score_select(xd["q"], xd["k"], cfg.K, noise=xd["noise"])
    sel2 = sas.select(s_gpu, cfg.K)
    assert torch.equal(idx, sel2[0]) and torch.equal(cnt, sel2[1])
    assert torch.equal(lg, sel2[2]) and torch.equal(lse_s, sel2[3])
    o, lse = sas.attn_fwd(xd["q"], xd["k"], xd["v"], idx, cnt, lg, sc)
    sas.attn_bwd(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, s_gpu, lse_s, idx, cnt, lg, sc)
    torch.cuda.synchronize()
    sas.get_error_flag()


def _check_rows(s_ref_rows, nh_rows, gidx, gcnt, glg, glse, sg_rows, K, name):
    """Selection of each row against the oracle's on the oracle's scores (see module doc)."""
    for r, (row, nh) in enumerate(zip(s_ref_rows, nh_rows)):
        row = row[:nh]
        c = min(K, nh)
        assert int(gcnt[r]) == c, (name, r)
        if c == nh:
            assert list(gidx[r, :c]) == list(range(nh))
        elif c:
            srt = np.sort(row)[::-1]
            ref = O.topk_history(row, nh, K)
            if srt[c - 1] - srt[c] > 2 * SCORE_TOL:
                assert list(gidx[r, :c]) == ref, (name, r)
            else:
                g = gidx[r, :c]
                assert np.all(np.diff(g) > 0) and np.all(row[g] >= srt[c - 1] - 2 * SCORE_TOL)
        assert np.all(gidx[r, c:] == -1)
        if nh:
            lse_ref = O.logsumexp(row)
            assert abs(float(glse[r]) - lse_ref) <= SCORE_TOL * max(1.0, abs(lse_ref))
            if c:
                g = gidx[r, :c]
                assert np.max(np.abs(glg[r, :c] - (row[g] - lse_ref))) <= 2 * SCORE_TOL
                assert np.max(np.abs(glg[r, :c] - (sg_rows[r][g] - float(glse[r])))) <= 1e-5


@pytest.mark.parametrize("max_hist,K,G", [(24, 5, 4), (1024, 32, 4), (2048, 16, 5)])
def test_score_select_decode_against_oracle(max_hist, K, G):
    """Pooled-key cache + decode stand-in scores + decode selection, against the oracle's
    fp64 decode stand-in scores (which pool the pages themselves) and its Top-K."""
    cfg = inputs.DecodeConfig("dscore", N=3, Hq=2 * G, Hkv=2, D=128, K=K, min_hist=max_hist // 2,
                              max_hist=max_hist, partial=True, seed=max_hist + G)
    x = inputs.make_decode(cfg)
    x["kv_len"][0] = 1                                   # no history at all
    noise = torch.randn((cfg.N, cfg.Hkv, max_hist), generator=torch.Generator().manual_seed(7))
    xd = {k: v.cuda() for k, v in x.items()}
    kpool = sas.pool_pages(xd["k_cache"])
    s, idx, cnt, lg, lse_s = sas.score_select_decode(xd["q"], kpool, xd["page_table"], xd["kv_len"], K, max_hist,
                                                     noise=noise.cuda())
    torch.cuda.synchronize()
    sas.get_error_flag()
    # the pooled keys against the page means in fp64
    ref_pool = x["k_cache"].double().mean(dim=2)
    assert float((kpool.cpu().double() - ref_pool).abs().max()) <= 1e-6
    s_ref = O.standin_scores_decode(x["q"], x["k_cache"], x["page_table"], x["kv_len"], noise)
    nh = O.decode_history(x["kv_len"])
    sg = s.cpu().numpy().astype(np.float64)
    for n in range(cfg.N):
        if nh[n]:
            assert np.max(np.abs(sg[n, :, :nh[n]] - s_ref[n, :, :nh[n]])) <= SCORE_TOL
    rows = [(n, h) for n in range(cfg.N) for h in range(cfg.Hkv)]
    _check_rows([s_ref[n, h] for n, h in rows], [int(nh[n]) for n, _ in rows],
                *(t.cpu().numpy().reshape(len(rows), *t.shape[2:]) for t in (idx, cnt, lg, lse_s)),
                [sg[n, h] for n, h in rows], K, f"decode {max_hist}")


def test_pool_pages_listed_pages_only():
    """With a page list only those pages are pooled; a bad id is flagged and skipped."""
    g = torch.Generator().manual_seed(3)
    kc = torch.randn((10, 2, 64, 64), generator=g).to(torch.bfloat16).cuda()
    kpool = torch.full((10, 2, 64), 7.0, device="cuda")
    sas.get_error_flag()
    sas.pool_pages(kc, pages=torch.tensor([3, 12, 5], dtype=torch.int32, device="cuda"), kpool=kpool)
    with pytest.raises(sas.SasError):
        sas.get_error_flag()
    ref = kc.double().mean(dim=2)
    for p in range(10):
        if p in (3, 5):
            assert float((kpool[p].double() - ref[p]).abs().max()) <= 1e-6
        else:
            assert torch.all(kpool[p] == 7.0)
