"""Host-side arithmetic of bench.py, on CPU: the work counts behind `value`
and `roofline`, the guard on the recorded DRAM traffic, the clock-record
parser and the dk/dv load-balance model.

The tile counts are pinned to the figures derived by hand for the three
prefill workloads (sum over query blocks i of min(K, i) + 1 kept blocks, the
current one included, times the query heads and the batch), so a change in
how `value` counts work shows up here.
"""
import types

import numpy as np
import pytest
import torch

import bench
from trainable_gated_block_b200 import inputs


@pytest.mark.parametrize("name,tiles", [
    ("qwen3-8b-32k", 523_776),        # 32 heads x (1 + ... + 32 + 480 x 33)
    ("qwen3-4b-8k", 65_280),          # 32 heads x (1 + ... + 16 + 112 x 17)
    ("qwen3-14b-2x32k", 365_760),     # 2 x 40 heads x (1 + ... + 8 + 504 x 9)
])
def test_prefill_tiles(name, tiles):
    cfg = inputs.workload(name)
    assert bench.prefill_tiles(cfg) == tiles


def test_prefill_flops_of_the_headline_workload():
    cfg = inputs.workload("qwen3-8b-32k")
    flops = 14 * 64 * 64 * cfg.D * bench.prefill_tiles(cfg)
    assert abs(flops - 3.8445e12) < 1e8
    # whole-job throughput: every replica's flops over the slowest rank's time
    assert bench.weak_tflops(1, flops, 6.0) == pytest.approx(640.75, rel=1e-4)
    assert bench.weak_tflops(4, flops, 6.0) == pytest.approx(4 * 640.75, rel=1e-4)


def test_decode_bytes_small_case():
    cfg = types.SimpleNamespace(N=2, Hq=4, Hkv=2, D=128, K=3)
    kv_len = torch.tensor([65, 200])       # current blocks hold 1 and 8 tokens
    cnt = torch.tensor([[1, 1], [3, 2]])   # kept history blocks per (sequence, KV head)
    tokens = (1 * 64 + 1) * 2 + (3 * 64 + 8) + (2 * 64 + 8)
    kv = tokens * 128 * 2 * 2              # K and V, bf16
    qo = 2 * 4 * 128 * 2 * 2               # q in, o out
    sel = 2 * 2 * (3 * 8 + 4) + (2 + 2 + 4 + 3) * 4 + 2 * 4
    assert bench.decode_bytes(cfg, kv_len, cnt) == kv + qo + sel


def test_select_bytes():
    assert bench.select_bytes(100, 10, 4) == 100 * 4 + 10 * (4 * 8 + 8)


def test_recorded_traffic_follows_the_source_hash(monkeypatch):
    entry = "sas_attn_bwd"
    rec = bench.DRAM_TRAFFIC["qwen3-8b-32k"][entry]
    assert rec[1] == bench.sources_hash(entry)          # recorded on the current sources
    assert bench.recorded_traffic("qwen3-8b-32k", entry) == rec[0]
    stale = {"qwen3-8b-32k": {entry: (rec[0], "0" * 16)}}
    monkeypatch.setattr(bench, "DRAM_TRAFFIC", stale)
    assert bench.recorded_traffic("qwen3-8b-32k", entry) is None
    assert bench.recorded_traffic("no-such-workload", entry) is None


class _FakeSmi:
    """Stands in for the nvidia-smi process: returns canned CSV lines."""

    def __init__(self, lines):
        self.lines = lines

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return "\n".join(self.lines) + "\n", ""


def test_clock_record_parsing():
    c = bench.ClockSampler("GPU-fake")
    c.proc = _FakeSmi([
        "1965, 1965, 700.1, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, 990.0, Not Active, Not Active, Not Active, Active",
        "1965, 1965, 980.5, Not Active, Not Active, Not Active, Not Active",
        "[N/A], 1965, 0.0, Not Active, Not Active, Not Active, Not Active",   # unreadable sample
    ])
    rec = c.stop()
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    c2 = bench.ClockSampler("GPU-fake")
    assert c2.stop()["reasons"] == ["clock sampling unavailable"]


def test_dkv_balance_model():
    # one (b, h), four key blocks; query blocks 1..3 keep block 0, query block 3 also keeps 1
    idx = np.full((1, 4, 2), -1)
    idx[0, 1] = [0, -1]
    idx[0, 2] = [0, -1]
    idx[0, 3] = [0, 1]
    r = bench._dkv_balance(idx, 4, 1, 2)
    # steps per key block: 1 + (times kept) = [4, 2, 1, 1]; longest first, snake over 2 CTAs:
    # round 0: CTA0 <- 4, CTA1 <- 2; round 1 (reversed): CTA1 <- 1, CTA0 <- 1
    assert r["items"] == 4 and r["steps_max_item"] == 4
    assert r["cta_steps_max"] == 5 and r["cta_steps_mean"] == 4.0
    assert r["cta_max_over_mean"] == 1.25


@pytest.mark.parametrize("name,gflop", [
    ("qwen3-8b-32k", 3785.3),       # the causal-exact counts of the scope table
    ("qwen3-4b-8k", 464.4),
    ("qwen3-14b-2x32k", 2536.7),
])
def test_prefill_causal_flops(name, gflop):
    cfg = inputs.workload(name)
    assert abs(bench.prefill_causal_flops(cfg) / 1e9 - gflop) < 0.06
    # a partial last block: the tile count rounds it up, the causal count does not
    small = inputs.PrefillConfig("p", "bf16", 1, 100, 2, 1, 128, 1, "normal", 1.0, seed=1)
    pairs = (64 * 65 // 2) + (1 * 64 * 36 + 36 * 37 // 2)     # block 0; block 1 (36 rows, 1 kept block)
    assert bench.prefill_causal_flops(small) == 14 * 128 * pairs * 2
