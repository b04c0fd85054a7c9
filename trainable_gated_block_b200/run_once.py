"""Run the path on one named workload a few times, for profilers.

    python -m trainable_gated_block_b200.run_once --workload qwen3-4b-8k --reps 2
    python -m trainable_gated_block_b200.run_once --workload decode-64seq --reps 2
    python -m trainable_gated_block_b200.run_once --workload decode-64seq --seqs 16 --reps 1
    python -m trainable_gated_block_b200.run_once --workload qwen3-8b-32k --part score --reps 2
    python -m trainable_gated_block_b200.run_once --workload qwen3-4b-8k --full-history --reps 1
    python -m trainable_gated_block_b200.run_once --decode-ctx 524288 --seqs 1 --reps 2

A prefill workload runs select -> forward -> backward; a decode workload runs
select -> paged decode. Nothing is timed or checked here: this is the command
that ncu captures wrap (the numbers come from bench.py and the checks from
the tests). ``--seqs`` keeps the first sequences of a decode workload only,
so that a full capture holds a few GB on the device.
"""
from __future__ import annotations

import argparse
import dataclasses
import math

import torch

from trainable_gated_block_b200 import build, inputs, sas


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="qwen3-4b-8k")
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--seqs", type=int, default=0, help="decode: use this many sequences")
    ap.add_argument("--part", default="path", choices=["path", "score"])
    ap.add_argument("--full-history", action="store_true")
    ap.add_argument("--decode-ctx", type=int, default=0)
    ap.add_argument("--dense", action="store_true")
    a = ap.parse_args()
    build.build()
    if a.decode_ctx:
        N, Hq, Hkv, D, K = a.seqs or 1, 32, 8, 128, 32
        x = inputs.make_decode_device(N, a.decode_ctx, Hq, Hkv, D, seed=1, device="cuda")
        nh = a.decode_ctx // 64
        Kd = nh if a.dense else K
        ws = torch.empty(max(256, sas.decode_workspace_bytes(N, Hq, Hkv, D, Kd)), dtype=torch.uint8, device="cuda")
        for _ in range(a.reps):
            sel = sas.select(x["s"], Kd, kv_len=x["kv_len"])
            sas.decode_paged(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["kv_len"], *sel[:3],
                             workspace=ws, with_lse=False)
        torch.cuda.synchronize()
        sas.get_error_flag()
        print(f"ran decode ctx={a.decode_ctx} x{a.reps}")
        return
    cfg = inputs.workload(a.workload)
    if a.full_history:
        cfg = dataclasses.replace(cfg, K=cfg.NQB)
    if a.seqs and isinstance(cfg, inputs.DecodeConfig):
        cfg = dataclasses.replace(cfg, N=a.seqs)
    if isinstance(cfg, inputs.DecodeConfig):
        x = {k: v.cuda() for k, v in inputs.make_decode(cfg).items()}
        ws = torch.empty(sas.decode_workspace_bytes(cfg.N, cfg.Hq, cfg.Hkv, cfg.D, cfg.K), dtype=torch.uint8,
                         device="cuda")
        for _ in range(a.reps):
            sel = sas.select(x["s"], cfg.K, kv_len=x["kv_len"])
            sas.decode_paged(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["kv_len"], *sel[:3],
                             workspace=ws, with_lse=False)
    elif a.part == "score":
        x = {k: v.cuda() for k, v in inputs.make_prefill(cfg, with_do=False).items()}
        for _ in range(a.reps):
            sas.score_select(x["q"], x["k"], cfg.K, noise=x.get("noise"))
    else:
        x = {k: v.cuda() for k, v in inputs.make_prefill(cfg).items()}
        sc = 1.0 / math.sqrt(cfg.D)
        ws = torch.empty(sas.bwd_workspace_bytes(x["q"], x["k"], cfg.K), dtype=torch.uint8, device="cuda")
        for _ in range(a.reps):
            sel = sas.select(x["s"], cfg.K)
            o, lse = sas.attn_fwd(x["q"], x["k"], x["v"], *sel[:3], sc)
            sas.attn_bwd(x["q"], x["k"], x["v"], o, x["do"], lse, x["s"], sel[3], sel[0], sel[1], sel[2], sc,
                         workspace=ws)
    torch.cuda.synchronize()
    sas.get_error_flag()
    print(f"ran {a.workload} x{a.reps}")


if __name__ == "__main__":
    main()
