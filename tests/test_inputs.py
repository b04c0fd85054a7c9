"""The seeded input generators (CPU): shapes, dtypes, determinism, and the
structure the workloads promise (the paged decode layout, the packed batch).
They hold none of the method's arithmetic; these checks make sure the
oracle and the kernels are fed what the workload recipes say."""
import torch

from trainable_gated_block_b200 import inputs


def test_prefill_shapes_dtypes_and_determinism():
    cfg = inputs.PrefillConfig("t", "bf16", 2, 200, 8, 2, 128, 3, "normal", 2.0, seed=5)
    a, b = inputs.make_prefill(cfg), inputs.make_prefill(cfg)
    assert a["q"].shape == (2, 200, 8, 128) and a["k"].shape == (2, 200, 2, 128) and a["v"].shape == (2, 200, 2, 128)
    assert a["q"].dtype == torch.bfloat16 and a["s"].dtype == torch.float32
    assert a["s"].shape == (2, 2, 4, 4)                          # ceil(200 / 64) blocks
    assert a["do"].shape == a["q"].shape
    for k in a:
        assert torch.equal(a[k], b[k]), k                        # same seed, same bits
    c = inputs.make_prefill(cfg, seed=6)
    assert not torch.equal(a["q"], c["q"])
    # scores drawn with the stated standard deviation (2.0 here)
    big = inputs.make_prefill(inputs.PrefillConfig("t", "bf16", 1, 64 * 64, 2, 1, 64, 3, "normal", 2.0, seed=1),
                              with_do=False)
    assert abs(float(big["s"].std()) - 2.0) < 0.05


def test_decode_layout():
    cfg = inputs.DecodeConfig("t", N=16, Hq=8, Hkv=2, D=128, K=4, min_hist=2, max_hist=20, partial=True, seed=9)
    x = inputs.make_decode(cfg)
    kv_len, pt = x["kv_len"].to(torch.int64), x["page_table"].to(torch.int64)
    assert x["q"].shape == (16, 8, 128) and x["s"].shape == (16, 2, 20)
    hist, cur = (kv_len - 1) // 64, kv_len - 64 * ((kv_len - 1) // 64)
    assert bool(((hist >= 2) & (hist <= 20)).all()) and bool(((cur >= 1) & (cur <= 64)).all())
    pages = (kv_len + 63) // 64
    used = torch.cat([pt[n, :int(pages[n])] for n in range(16)])
    total = x["k_cache"].shape[0]
    assert total == int(pages.sum()) == x["v_cache"].shape[0]
    assert torch.equal(torch.sort(used).values, torch.arange(total))   # every page used exactly once
    assert x["k_cache"].shape[1:] == (2, 64, 128)
    # not all sequences' pages are contiguous: the permutation scatters them
    assert any(bool((pt[n, 1:int(pages[n])] - pt[n, :int(pages[n]) - 1] != 1).any()) for n in range(16))


def test_decode_one_token_current_block():
    cfg = inputs.DecodeConfig("t", N=8, Hq=4, Hkv=1, D=128, K=2, min_hist=3, max_hist=9, seed=2)
    x = inputs.make_decode(cfg)
    kv_len = x["kv_len"].to(torch.int64)
    assert bool(((kv_len - 1) % 64 == 0).all())                  # history in whole blocks + 1 new token


def test_varlen_packing():
    lengths = [100, 64, 1, 229, 0, 130]
    x = inputs.make_varlen(lengths, 4, 2, 128, "bf16", 1.0, seed=3)
    cu = x["cu_seqlens"].to(torch.int64)
    assert cu.tolist() == [0, 100, 164, 165, 394, 394, 524]
    T = 524
    assert x["q"].shape == (T, 4, 128) and x["k"].shape == (T, 2, 128)
    nqb = (229 + 63) // 64
    assert x["s"].shape[0] == len(lengths) and x["s"].shape[2] >= nqb
