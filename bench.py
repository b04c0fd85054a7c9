#!/usr/bin/env python
"""Benchmark of the SAS gated block-sparse attention hot path on B200.

One step = the whole path on one batch of seeded synthetic input:
  prefill/training part on the Qwen3-8B-shaped 32k layer (B=1, S=32768,
  32/8 heads, D=128, K=32): select -> forward -> backward (dq, dk, dv, ds);
  decode part on 64 paged sequences (8k..64k context, 32/8 heads, K=32):
  select -> paged decode.
`value` is the prefill part's throughput in TFLOPS counting only attended
64x64 tiles (14*64*64*D flops per tile: 4 forward, 10 backward) over the
device time of select+forward+backward. Decode is reported beside it in GB/s
of algorithmic HBM bytes and tokens/s.

Multi-GPU (torchrun): every rank runs its own independent replica of the
workload (different seed), no collective in the data path; the timed region
is bracketed by barriers and the max over ranks is reported (weak scaling).

Beside that headline line, after the timed steps (rank 0 prints them as extra
keys of the same JSON line): the Qwen3-4B 8k and Qwen3-14B 2x32k layers
(`configs`), the full-history variant (K >= #history) of the 32k layer with
its dk/dv load balance (`full_history`), the stand-in scorer + select in one
call (`score_select`), and a decode scaling study over 64K-512K of context at batch
1 and 8, sparse against the same kernel reading every block (`decode_scaling`,
CUDA-graph replays). Every extra number is the median of CUDA-event times of
back-to-back CUDA-graph replays (so short calls carry no host launch gaps; a
small call's inputs may then sit in L2).

`--impl reference` times the fp64 CPU oracle instead (rank 0 only), each
step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

BLOCK = 64
L2_BYTES = 126 * 2**20


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefill", default="qwen3-8b-32k")
    ap.add_argument("--decode", default="decode-64seq")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample budget")
    ap.add_argument("--no-extras", action="store_true", help="skip the extra configs and studies")
    return ap.parse_args()


def _peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return dict(hbm=float(m["hbm_gbs"]), bf16=float(m["bf16_tflops"]),
                    bf16_sustained=float(m.get("bf16_tflops_sustained", m["bf16_tflops"])), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------------------
# replicas: one process per GPU, no collective in the data path
# ---------------------------------------------------------------------------

def rank_env():
    """(world size, rank, local rank) as torchrun sets them; one process without it."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(base, rank):
    """Each rank runs its own replica of the workload on its own seeded inputs."""
    return base + 1000 * rank


def max_over_ranks(vals, dist, device):
    """Element-wise max of per-rank timings over the process group (the slowest
    rank sets the job's time); the values unchanged in a single process."""
    vals = [float(v) for v in vals]
    if dist is None or not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    import torch
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def weak_tflops(world, flops_per_replica, ms):
    """Whole-job throughput: the flops of every replica over the slowest rank's time."""
    return world * flops_per_replica / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# work counts (algorithmic)
# ---------------------------------------------------------------------------

def prefill_tiles(cfg):
    """Attended 64x64 tiles over all query heads: sum over query blocks of (min(K, i) + 1)."""
    per_head = sum(min(cfg.K, i) + 1 for i in range(cfg.NQB))
    return per_head * cfg.B * cfg.Hq


def prefill_causal_flops(cfg):
    """The causal-exact count: 14 D flops per (query, key) pair actually attended,
    64 x rows for a kept history block and the causal triangle rows (rows + 1) / 2
    for the query block's own block (rows = 64, or fewer for a partial last block)."""
    per_head = 0
    for i in range(cfg.NQB):
        rows = min(BLOCK, cfg.S - i * BLOCK)
        per_head += min(cfg.K, i) * BLOCK * rows + rows * (rows + 1) // 2
    return 14 * cfg.D * per_head * cfg.B * cfg.Hq


def decode_bytes(cfg, kv_len, cnt):
    """Algorithmic HBM bytes of one decode call: kept K/V pages (full history
    pages, the current block's valid tokens), q, o, selection and page ids."""
    import torch
    kv_len = kv_len.to(torch.int64).cpu()
    cnt = cnt.to(torch.int64).cpu()                       # [N, Hkv]
    c = (kv_len - 1) // BLOCK
    cur_tokens = (kv_len - c * BLOCK)[:, None]             # [N, 1]
    tokens = cnt * BLOCK + cur_tokens                      # [N, Hkv]
    kv = int(tokens.sum()) * cfg.D * 2 * 2
    qo = cfg.N * cfg.Hq * cfg.D * 2 * 2
    sel = cfg.N * cfg.Hkv * (cfg.K * 8 + 4) + int((cnt + 1).sum()) * 4 + cfg.N * 4
    return kv + qo + sel


def select_bytes(nh_total, rows, K):
    return nh_total * 4 + rows * (K * 8 + 8)


# ---------------------------------------------------------------------------
# DRAM bytes (read + write) per call of each entry point, summed over its
# kernels, from one `ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum`
# capture of run_once on the workload. Each figure carries the hash of the
# kernel sources it was taken on; when the sources change the figure is no
# longer reported (traffic: null) until it is captured again.
# ---------------------------------------------------------------------------
TRAFFIC_SOURCES = {
    "sas_attn_fwd": ["attn_fwd_sm100.cu", "sm100.cuh", "common.cuh"],
    "sas_attn_bwd": ["attn_bwd_sm100.cu", "attn_simt.cu", "sm100.cuh", "common.cuh"],
}
DRAM_TRAFFIC = {
    # workload -> entry point -> (bytes per call, sha256[:16] of the sources above);
    # the backward's figure sums Dr, dq and dk/dv (its index and ds kernels, about
    # 40 MB, are not in the capture)
    "qwen3-8b-32k": {
        "sas_attn_fwd": (641328128, "a313d0a8f00a589c"),
        "sas_attn_bwd": (5719122176, "05516f899d0d18c8"),
    },
}


def sources_hash(entry):
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES[entry]:
        with open(os.path.join(HERE, "trainable_gated_block_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, entry):
    """DRAM bytes per call recorded for the current kernel sources, else None."""
    rec = DRAM_TRAFFIC.get(workload, {}).get(entry)
    if rec is None or entry not in TRAFFIC_SOURCES or rec[1] != sources_hash(entry):
        return None
    return rec[0]


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}",
                   "--format=csv,noheader,nounits", "-lms", "20"]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["clock sampling unavailable"], samples=0)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return dict(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=max(mx) if mx else None,
                    reasons=sorted(reasons), samples=len(sm))


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def run_ours(a):
    import torch
    import torch.distributed as dist

    from trainable_gated_block_b200 import build, inputs, sas

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=torch.device("cuda", local))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    sas.lib()
    dev = torch.device("cuda", local)
    peaks = _peaks()

    pc = inputs.workload(a.prefill)
    dc = inputs.workload(a.decode)
    px = inputs.make_prefill(pc, seed=replica_seed(pc.seed, rank))
    dx = inputs.make_decode(dc, seed=replica_seed(dc.seed, rank))
    P = {k: v.to(dev) for k, v in px.items()}
    Dd = {k: v.to(dev) for k, v in dx.items()}
    sc_p = 1.0 / math.sqrt(pc.D)
    ws_b = torch.empty(sas.bwd_workspace_bytes(P["q"], P["k"], pc.K), dtype=torch.uint8, device=dev)
    ws_d = torch.empty(sas.decode_workspace_bytes(dc.N, dc.Hq, dc.Hkv, dc.D, dc.K), dtype=torch.uint8, device=dev)

    names = ["select", "fwd", "bwd", "dselect", "decode"]

    def step(rec):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)] if rec else None
        if rec:
            ev[0].record()
        sel = sas.select(P["s"], pc.K)
        if rec:
            ev[1].record()
        o, lse = sas.attn_fwd(P["q"], P["k"], P["v"], sel[0], sel[1], sel[2], sc_p)
        if rec:
            ev[2].record()
        grads = sas.attn_bwd(P["q"], P["k"], P["v"], o, P["do"], lse, P["s"], sel[3], sel[0], sel[1], sel[2],
                             sc_p, workspace=ws_b)
        if rec:
            ev[3].record()
        dsel = sas.select(Dd["s"], dc.K, kv_len=Dd["kv_len"])
        if rec:
            ev[4].record()
        od, _ = sas.decode_paged(Dd["q"], Dd["k_cache"], Dd["v_cache"], Dd["page_table"], Dd["kv_len"],
                                 dsel[0], dsel[1], dsel[2], workspace=ws_d, with_lse=False)
        if rec:
            ev[5].record()
        return ev, (o, grads, od, dsel)

    for _ in range(a.warmup):
        step(False)
    torch.cuda.synchronize()
    sas.get_error_flag()
    _, (_, _, _, dsel) = step(False)
    dec_bytes = decode_bytes(dc, dx["kv_len"], dsel[1])
    torch.cuda.synchronize()

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    launches0 = sas.kernel_launches()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    evs = [step(True)[0] for _ in range(a.steps)]
    t1.record()
    torch.cuda.synchronize()
    launches = sas.kernel_launches() - launches0
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    sas.get_error_flag()
    total_ms = t0.elapsed_time(t1)
    part_ms = {n: statistics.median(e[i].elapsed_time(e[i + 1]) for e in evs) for i, n in enumerate(names)}
    prefill_ms = part_ms["select"] + part_ms["fwd"] + part_ms["bwd"]
    dec_ms = part_ms["dselect"] + part_ms["decode"]
    t = max_over_ranks([total_ms, prefill_ms, dec_ms] + [part_ms[n] for n in names], dist, dev)
    total_ms, prefill_ms, dec_ms = t[0], t[1], t[2]
    part_ms = {n: t[3 + i] for i, n in enumerate(names)}

    tiles = prefill_tiles(pc)
    unit_flops = 64 * 64 * pc.D
    flops_fb = 14 * unit_flops * tiles
    tflops = weak_tflops(world, flops_fb, prefill_ms)
    bwd_tf = 10 * unit_flops * tiles / (part_ms["bwd"] * 1e-3) / 1e12
    fwd_tf = 4 * unit_flops * tiles / (part_ms["fwd"] * 1e-3) / 1e12
    dec_gbs = dec_bytes / (part_ms["decode"] * 1e-3) / 1e9
    nh_pre = sum(range(pc.NQB)) * pc.B * pc.Hkv
    sel_bytes = select_bytes(nh_pre, pc.B * pc.Hkv * pc.NQB, pc.K)
    sel_gbs = sel_bytes / (part_ms["select"] * 1e-3) / 1e9
    tag = "of measured" if peaks["source"] == "measured" else "of fallback"
    # tensor-core denominator: the burst bf16 GEMM figure while the SM clock stayed
    # near its maximum during the timed region (a ~10 ms step does not reach the
    # power cap), the sustained one if it dropped
    at_max = bool(clk.get("sm_mhz") and clk.get("sm_max_mhz") and clk["sm_mhz"] >= 0.9 * clk["sm_max_mhz"])
    tpeak = peaks["bf16"] if at_max else peaks["bf16_sustained"]
    tnote = "burst bf16, SM clock at max" if at_max else "sustained bf16"
    kernels = {
        "select": dict(bound="hbm", achieved=sel_gbs, peak=peaks["hbm"], unit="GB/s", frac=sel_gbs / peaks["hbm"],
                       ms=part_ms["select"], bytes=sel_bytes),
        "fwd": dict(bound="tensor", achieved=fwd_tf, peak=tpeak, unit="TFLOP/s", frac=fwd_tf / tpeak,
                    ms=part_ms["fwd"]),
        "bwd": dict(bound="tensor", achieved=bwd_tf, peak=tpeak, unit="TFLOP/s", frac=bwd_tf / tpeak,
                    ms=part_ms["bwd"]),
        "prefill": dict(bound="tensor", achieved=tflops / world, peak=tpeak, unit="TFLOP/s",
                        frac=tflops / world / tpeak, ms=prefill_ms),
        "decode": dict(bound="hbm", achieved=dec_gbs, peak=peaks["hbm"], unit="GB/s", frac=dec_gbs / peaks["hbm"],
                       ms=part_ms["decode"], bytes=dec_bytes, tokens_per_s=dc.N / (part_ms["decode"] * 1e-3)),
    }
    dom = max(("fwd", "bwd", "decode", "select"), key=lambda n: part_ms[n])
    kd = kernels[dom]
    traffic = recorded_traffic(pc.name, f"sas_{'attn_' if dom in ('fwd', 'bwd') else ''}{dom}")
    roofline = dict(bound=kd["bound"], achieved=round(kd["achieved"], 3), peak=kd["peak"], unit=kd["unit"],
                    frac=round(kd["frac"], 4), traffic=traffic, kernel=f"sas_{'attn_' if dom in ('fwd', 'bwd') else ''}{dom}",
                    peak_note=f"{tag} ({tnote if kd['bound'] == 'tensor' else 'HBM copy'})")

    e2e = None
    if not a.no_e2e:
        e2e = run_e2e(a, torch, sas, px, dx, P, Dd, pc, dc, sc_p, ws_b, ws_d, flops_fb, world, dist, dev)
    extras = {}
    if rank == 0 and not a.no_extras:
        extras = run_extras(torch, sas, inputs, P, px, pc, dev, peaks, tpeak, a)

    line = None
    if rank == 0:
        line = {
            "metric": "SAS gated block-sparse attn fwd+bwd TFLOPS & decode HBM GB/s vs roofline",
            "value": round(tflops, 3), "unit": "TFLOPS", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": round(total_ms / a.steps, 4), "higher_is_better": True, "scaling": "weak",
            "value_causal_exact": round(weak_tflops(world, prefill_causal_flops(pc), prefill_ms), 3),
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) q/k/v/dO, pooled stand-in scores)",
            "config": {
                "workload": f"{pc.name} select+fwd+bwd, then {dc.name} select+paged decode",
                "prefill": dict(B=pc.B, S=pc.S, Hq=pc.Hq, Hkv=pc.Hkv, D=pc.D, K=pc.K, block=BLOCK,
                                attended_tiles=tiles, flops_per_step=flops_fb,
                                flops_per_step_causal_exact=prefill_causal_flops(pc)),
                "decode": dict(N=dc.N, Hq=dc.Hq, Hkv=dc.Hkv, D=dc.D, K=dc.K, ctx="8k..64k",
                               algorithmic_bytes=dec_bytes),
                "l2": "inputs larger than L2 (prefill q/k/v/o/dO about 0.9 GB, decode pages 0.54 GB per step)",
                "parallelism": f"replicas x{world} (no collective)",
            },
            "decode": dict(gbs=round(dec_gbs, 1), tokens_per_s=round(world * dc.N / (dec_ms * 1e-3), 1),
                           us_decode_kernel=round(part_ms["decode"] * 1e3, 2), us_select=round(part_ms["dselect"] * 1e3, 2),
                           frac_hbm=round(dec_gbs / peaks["hbm"], 4)),
            "part_ms": {k: round(v, 4) for k, v in part_ms.items()},
            "kernels": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                        for k, v in kernels.items()},
            "roofline": roofline,
            "clocks": clk,
            "gpu_launches": launches,
            "e2e": e2e,
        }
        line.update(extras)
        if world == 1 and not a.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(pc, px, a.cpu_seconds)
            if not a.no_extras:
                # the oracle on the other two prefill workloads (fewer stripes each)
                per = {pc.name: dict(tflops=line["cpu_baseline"]["value"],
                                     parts_s=line["cpu_baseline"]["parts_s"])}
                for name in ("qwen3-4b-8k", "qwen3-14b-2x32k"):
                    cfg = inputs.workload(name)
                    cb = cpu_baseline(cfg, inputs.make_prefill(cfg), a.cpu_seconds / 3)
                    per[name] = dict(tflops=cb["value"], parts_s=cb["parts_s"], sample=cb["sample"])
                line["cpu_baseline"]["per_config"] = per
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line))


# ---------------------------------------------------------------------------
# extra measurements (rank 0, after the timed steps)
# ---------------------------------------------------------------------------

def _graph(torch, fns):
    """Capture the callables (run once eagerly first) into one CUDA graph."""
    for fn in fns:
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        for fn in fns:
            fn()
    return g


def _replay_ms(torch, g, reps=20, warmup=3):
    """Median device time (ms) of back-to-back replays of graph g (no host gap between
    them, so short calls are not padded by launch overhead)."""
    for _ in range(warmup):
        g.replay()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record()
    for k in range(reps):
        g.replay()
        ev[k + 1].record()
    torch.cuda.synchronize()
    return statistics.median(ev[k].elapsed_time(ev[k + 1]) for k in range(reps))


def _prefill_parts(torch, sas, P, cfg, K, ws, reps, warmup):
    """Median replay time of select, forward and backward, each captured in its own graph."""
    sc = 1.0 / math.sqrt(cfg.D)
    st = {}

    def sel():
        st["sel"] = sas.select(P["s"], K)

    def fwd():
        st["o"] = sas.attn_fwd(P["q"], P["k"], P["v"], *st["sel"][:3], sc)

    def bwd():
        sl = st["sel"]
        sas.attn_bwd(P["q"], P["k"], P["v"], st["o"][0], P["do"], st["o"][1], P["s"], sl[3], sl[0], sl[1], sl[2], sc,
                     workspace=ws)

    graphs = [(n, _graph(torch, [fn])) for n, fn in (("select", sel), ("fwd", fwd), ("bwd", bwd))]
    ms = {n: _replay_ms(torch, g, reps, warmup) for n, g in graphs}
    del graphs
    return ms, st


def _prefill_line(cfg, K, ms, tpeak, hbm):
    tiles = sum(min(K, i) + 1 for i in range(cfg.NQB)) * cfg.B * cfg.Hq
    unit = 64 * 64 * cfg.D
    pre = ms["select"] + ms["fwd"] + ms["bwd"]
    tf = lambda f, t: f * unit * tiles / (t * 1e-3) / 1e12          # noqa: E731
    return dict(B=cfg.B, S=cfg.S, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, K=K, attended_tiles=tiles,
                ms={k: round(v, 4) for k, v in ms.items()},
                tflops_prefill=round(tf(14, pre), 2), frac_prefill=round(tf(14, pre) / tpeak, 4),
                tflops_fwd=round(tf(4, ms["fwd"]), 2), frac_fwd=round(tf(4, ms["fwd"]) / tpeak, 4),
                tflops_bwd=round(tf(10, ms["bwd"]), 2), frac_bwd=round(tf(10, ms["bwd"]) / tpeak, 4))


def _dkv_balance(idx, NQB, n_bh, ctas):
    """Steps per CTA of the dk/dv kernel's deal, modelled on the host from the selection
    (items = key blocks; a key block's steps = its own block + every query block that kept
    it; longest first within a head, dealt in snake order over the CTAs): max / mean."""
    import numpy as np
    steps = np.ones((n_bh, NQB), dtype=np.int64)                  # own block
    for bh in range(n_bh):
        sel = idx[bh][idx[bh] >= 0]
        steps[bh] += np.bincount(sel.ravel(), minlength=NQB)[:NQB]
    order = [(bh, int(j)) for bh in range(n_bh) for j in np.argsort(-steps[bh], kind="stable")]
    per = np.zeros(ctas, dtype=np.int64)
    for pos, (bh, j) in enumerate(order):
        r, c = divmod(pos, ctas)
        per[c if r % 2 == 0 else ctas - 1 - c] += steps[bh, j]
    return dict(items=len(order), steps_max_item=int(steps.max()), steps_mean_item=round(float(steps.mean()), 2),
                cta_steps_max=int(per.max()), cta_steps_mean=round(float(per.mean()), 2),
                cta_max_over_mean=round(float(per.max() / per.mean()), 4))


def run_extras(torch, sas, inputs, P, px, pc, dev, peaks, tpeak, a):
    out = {}
    warmup = 2
    # --- the other two prefill workloads
    cfgs = {}
    for name in ("qwen3-4b-8k", "qwen3-14b-2x32k"):
        cfg = inputs.workload(name)
        x = {k: v.to(dev) for k, v in inputs.make_prefill(cfg).items()}
        ws = torch.empty(sas.bwd_workspace_bytes(x["q"], x["k"], cfg.K), dtype=torch.uint8, device=dev)
        ms, _ = _prefill_parts(torch, sas, x, cfg, cfg.K, ws, 10, warmup)
        cfgs[name] = _prefill_line(cfg, cfg.K, ms, tpeak, peaks["hbm"])
        del x, ws
        torch.cuda.empty_cache()
    out["configs"] = cfgs
    # --- the full-history variant on the headline workload's tensors
    Kf = pc.NQB
    ws = torch.empty(sas.bwd_workspace_bytes(P["q"], P["k"], Kf), dtype=torch.uint8, device=dev)
    ms, st = _prefill_parts(torch, sas, P, pc, Kf, ws, 3, 1)
    fh = _prefill_line(pc, Kf, ms, tpeak, peaks["hbm"])
    import numpy as np
    idx = st["sel"][0].cpu().numpy().reshape(pc.B * pc.Hkv, pc.NQB, Kf)
    fh["dkv_balance"] = _dkv_balance(idx, pc.NQB, pc.B * pc.Hkv,
                                     torch.cuda.get_device_properties(dev).multi_processor_count)
    out["full_history"] = {pc.name: fh}
    del ws, st
    torch.cuda.empty_cache()
    # --- stand-in scorer + select on the headline workload (its scores are the stand-in)
    if "noise" in px:
        noise = px["noise"].to(dev)
        s_buf = torch.zeros_like(P["s"])
        wsc = torch.empty(max(256, int(sas.lib().sas_score_select_workspace_size(pc.B, pc.S, pc.Hq, pc.Hkv, pc.D))),
                          dtype=torch.uint8, device=dev)
        g = _graph(torch, [lambda: sas.score_select(P["q"], P["k"], pc.K, noise=noise, workspace=wsc, s_out=s_buf)])
        ms = {"score_select": _replay_ms(torch, g, 20, 3)}
        del g
        rows = pc.B * pc.Hkv * pc.NQB
        nbytes = (P["q"].numel() + P["k"].numel()) * 2 + noise.numel() // 2 * 4 + \
            sum(range(pc.NQB)) * pc.B * pc.Hkv * 4 + rows * (pc.K * 8 + 8)
        out["score_select"] = dict(workload=pc.name, us=round(ms["score_select"] * 1e3, 2), bytes=int(nbytes),
                                   gbs=round(nbytes / (ms["score_select"] * 1e-3) / 1e9, 1),
                                   frac_hbm=round(nbytes / (ms["score_select"] * 1e-3) / 1e9 / peaks["hbm"], 4),
                                   note="pooling reads q and k once; scores written once (lower triangle)")
        del s_buf, wsc, noise
    torch.cuda.empty_cache()
    # --- decode scaling study
    out["decode_scaling"] = decode_scaling(torch, sas, inputs, dev, peaks)
    return out


def decode_scaling(torch, sas, inputs, dev, peaks):
    """Sparse (select + decode, K = 32; and the same with the stand-in scores computed from
    the pooled-key cache first, `scored`) against the same decode kernel reading every block
    (K >= #history, selection given), at 64K-512K of context, batch 1 and 8. Each arm is
    captured in a CUDA graph and replayed; the median replay time is reported."""
    Hq, Hkv, D, K = 32, 8, 128, 32
    rows = []
    for batch in (1, 8):
        for ctx in (65536, 131072, 262144, 524288):
            x = inputs.make_decode_device(batch, ctx, Hq, Hkv, D, seed=ctx + batch, device=dev)
            nh = ctx // BLOCK
            ws_s = torch.empty(max(256, sas.decode_workspace_bytes(batch, Hq, Hkv, D, K)), dtype=torch.uint8,
                               device=dev)
            ws_d = torch.empty(max(256, sas.decode_workspace_bytes(batch, Hq, Hkv, D, nh)), dtype=torch.uint8,
                               device=dev)
            dense_idx = torch.arange(nh, dtype=torch.int32, device=dev).expand(batch, Hkv, nh).contiguous()
            dense_cnt = torch.full((batch, Hkv), nh, dtype=torch.int32, device=dev)
            dense_lg = torch.full((batch, Hkv, nh), -math.log(nh), dtype=torch.float32, device=dev)
            kpool = sas.pool_pages(x["k_cache"])      # pooled-key cache, filled once per page (not timed)
            st = {}

            def scored_sel():
                st["sel"] = sas.score_select_decode(x["q"], kpool, x["page_table"], x["kv_len"], K, nh)[1:]

            def sparse_sel():
                st["sel"] = sas.select(x["s"], K, kv_len=x["kv_len"])

            def sparse_dec():
                sas.decode_paged(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["kv_len"], *st["sel"][:3],
                                 workspace=ws_s, with_lse=False)

            def dense_dec():
                sas.decode_paged(x["q"], x["k_cache"], x["v_cache"], x["page_table"], x["kv_len"], dense_idx,
                                 dense_cnt, dense_lg, workspace=ws_d, with_lse=False)

            res = {}
            for arm, fns in (("sparse", [sparse_sel, sparse_dec]), ("scored", [scored_sel, sparse_dec]),
                             ("dense", [dense_dec])):
                g = _graph(torch, fns)
                res[arm] = _replay_ms(torch, g, 10, 2)
                del g
            for arm, fn in (("sparse_select", sparse_sel), ("scored_select", scored_sel)):
                g = _graph(torch, [fn])
                res[arm] = _replay_ms(torch, g, 10, 2)
                del g
            sas.get_error_flag()
            kv_sparse = batch * Hkv * (K * BLOCK + 1) * D * 2 * 2
            kv_dense = batch * Hkv * (nh * BLOCK + 1) * D * 2 * 2
            rows.append(dict(batch=batch, context=ctx, K=K,
                             us_sparse=round(res["sparse"] * 1e3, 2), us_sparse_select=round(res["sparse_select"] * 1e3, 2),
                             us_scored=round(res["scored"] * 1e3, 2),
                             us_scored_select=round(res["scored_select"] * 1e3, 2),
                             us_dense=round(res["dense"] * 1e3, 2), speedup=round(res["dense"] / res["sparse"], 2),
                             speedup_scored=round(res["dense"] / res["scored"], 2),
                             scoring_share=round(res["scored_select"] / res["scored"], 3),
                             dense_gbs=round(kv_dense / (res["dense"] * 1e-3) / 1e9, 1),
                             dense_frac_hbm=round(kv_dense / (res["dense"] * 1e-3) / 1e9 / peaks["hbm"], 4),
                             sparse_kv_bytes=kv_sparse, dense_kv_bytes=kv_dense))
            del x, ws_s, ws_d, dense_idx, dense_cnt, dense_lg, st, kpool
            torch.cuda.empty_cache()
    return dict(rows=rows, note="kernel-level time of one decode step (graph replay); the pages' 2.4x/4.6x/5.6x "
                                "(batch 1, 64K/256K/512K) and ~13x (batch 8, 64K) are whole-model serving latencies "
                                "on other hardware, quoted as context only")


def _pipelined(torch, hin, dsets, compute, steps, warmup, world, dist):
    """Steps through the public API with host copies in the timed region.

    Step n copies its inputs (`hin`, pinned host tensors) into the device set
    dsets[n % 2] on an input stream, runs compute(dset) -> {name: tensor} on the
    current stream and copies every result into pinned host buffers on an
    output stream, so the upload of step n + 1 and the download of step n - 1
    overlap the compute of step n. A device set is rewritten only after the
    compute that read it has finished. Returns the device time per step over
    `steps` steps (CUDA events on the current stream, which waits for the other
    two streams before the closing event) and the bytes read back per step."""
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    freed = [None, None]
    outs = [{}, {}]

    def step(n):
        b = dsets[n % 2]
        if freed[n % 2] is not None:
            s_in.wait_event(freed[n % 2])
        with torch.cuda.stream(s_in):
            for k, t in hin.items():
                b[k].copy_(t, non_blocking=True)
        comp.wait_stream(s_in)
        res = compute(b)
        freed[n % 2] = comp.record_event()
        s_out.wait_stream(comp)
        with torch.cuda.stream(s_out):
            for k, t in res.items():
                t.record_stream(s_out)
                if k not in outs[n % 2]:
                    outs[n % 2][k] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                outs[n % 2][k].copy_(t, non_blocking=True)

    for n in range(max(1, warmup)):
        step(n)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    s_in.wait_stream(comp)
    s_out.wait_stream(comp)
    for n in range(steps):
        step(n)
    comp.wait_stream(s_in)
    comp.wait_stream(s_out)
    t1.record()
    torch.cuda.synchronize()
    d2h = sum(t.numel() * t.element_size() for t in outs[0].values())
    return t0.elapsed_time(t1) / steps, d2h


def run_e2e(a, torch, sas, px, dx, P, Dd, pc, dc, sc_p, ws_b, ws_d, flops_fb, world, dist, dev):
    """The prefill step and the decode step through the public API, each step's
    inputs copied from pinned host memory and each step's results read back to
    pinned host memory inside the timed region (pipelined over three streams)."""
    hin_p = {k: px[k].pin_memory() for k in ("q", "k", "v", "do", "s")}
    hin_d = {k: dx[k].pin_memory() for k in ("q", "s", "kv_len", "page_table")}
    h2d_p = sum(t.numel() * t.element_size() for t in hin_p.values())
    h2d_d = sum(t.numel() * t.element_size() for t in hin_d.values())

    def prefill(b):
        sel = sas.select(b["s"], pc.K)
        o, lse = sas.attn_fwd(b["q"], b["k"], b["v"], sel[0], sel[1], sel[2], sc_p)
        dq, dk, dv, ds = sas.attn_bwd(b["q"], b["k"], b["v"], o, b["do"], lse, b["s"], sel[3], sel[0], sel[1],
                                      sel[2], sc_p, workspace=ws_b)
        return dict(o=o, dq=dq, dk=dk, dv=dv, ds=ds)

    def decode(b):
        dsel = sas.select(b["s"], dc.K, kv_len=b["kv_len"])
        od, _ = sas.decode_paged(b["q"], Dd["k_cache"], Dd["v_cache"], b["page_table"], b["kv_len"],
                                 dsel[0], dsel[1], dsel[2], workspace=ws_d, with_lse=False)
        return dict(od=od)

    sets_p = [{k: P[k] for k in hin_p}, {k: torch.empty_like(P[k]) for k in hin_p}]
    sets_d = [{k: Dd[k] for k in hin_d}, {k: torch.empty_like(Dd[k]) for k in hin_d}]
    pre, d2h_p = _pipelined(torch, hin_p, sets_p, prefill, a.steps, a.warmup, world, dist)
    dec, d2h_d = _pipelined(torch, hin_d, sets_d, decode, a.steps, a.warmup, world, dist)
    sas.get_error_flag()
    pre, dec = max_over_ranks([pre, dec], dist, dev)
    return dict(value=round(weak_tflops(world, flops_fb, pre), 3), unit="TFLOPS",
                h2d_bytes_per_step=int(h2d_p + h2d_d), d2h_bytes_per_step=int(d2h_p + d2h_d),
                ms_prefill=round(pre, 3), ms_decode=round(dec, 3),
                decode_tokens_per_s=round(world * dc.N / (dec * 1e-3), 1),
                overlap="upload of step n+1 and download of step n-1 run beside step n's kernels")


# ---------------------------------------------------------------------------
# the fp64 CPU oracle (the cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def _oracle_stripes(pc, px, budget_s, max_stripes=10**9, parts=None):
    """Time oracle forward+backward stripes of the workload until the budget is spent.

    Returns (attended-tile flops, stripes, seconds of fwd+bwd); if a dict is
    given as ``parts``, the seconds of select, fwd and bwd are added to it."""
    import numpy as np

    from oracle import sas_oracle as O
    # query head 0 and its KV head only (G = 1 view), so the oracle's full-size
    # output buffers stay small
    q, do = (O._f64(px[n][:1, :, :1]) for n in ("q", "do"))
    k, v = (O._f64(px[n][:1, :, :1]) for n in ("k", "v"))
    s = px["s"][:1, :1].numpy()
    rows = [pc.NQB - 1 - 7 * r for r in range(pc.NQB // 7)]      # spread over the sequence
    flops, n, t_spent = 0, 0, 0.0
    sc = 1.0 / math.sqrt(pc.D)
    for i in rows:
        if t_spent >= budget_s or n >= max_stripes:
            break
        s1 = s[:1, :1, i:i + 1, :]
        t_sel = time.perf_counter()
        idx1, cnt1, lg1, _ = O.select(s1, pc.K, np.array([[i]]))
        t_sel = time.perf_counter() - t_sel
        idx = np.full((1, 1, pc.NQB, pc.K), -1, dtype=np.int32)
        cnt = np.zeros((1, 1, pc.NQB), dtype=np.int32)
        lg = np.full((1, 1, pc.NQB, pc.K), -np.inf)
        idx[0, 0, i], cnt[0, 0, i], lg[0, 0, i] = idx1[0, 0, 0], cnt1[0, 0, 0], lg1[0, 0, 0]
        t0 = time.perf_counter()
        O.attn_fwd(q, k, v, idx, cnt, lg, sc, stripes=[(0, 0, i)])
        t1 = time.perf_counter()
        O.attn_bwd(q, k, v, do, idx, cnt, lg, s, sc, stripes=[(0, 0, i)])
        t2 = time.perf_counter()
        t_spent += t2 - t0
        if parts is not None:
            for name, dt in (("select", t_sel), ("fwd", t1 - t0), ("bwd", t2 - t1)):
                parts[name] = parts.get(name, 0.0) + dt
        flops += 14 * 64 * 64 * pc.D * (int(cnt[0, 0, i]) + 1)
        n += 1
    return flops, n, t_spent


def cpu_baseline(pc, px, budget_s):
    parts = {}
    flops, n, t = _oracle_stripes(pc, px, budget_s, parts=parts)
    return dict(value=flops / t / 1e12, unit="TFLOPS", cores=_blas_threads(), kind="oracle",
                sample=f"fp64 oracle forward+backward of {n} 64-row stripes (batch 0, head 0) of the "
                       f"{pc.name} workload, {t:.1f} s, counted as attended-tile flops",
                parts_s={k: round(v, 3) for k, v in parts.items()},
                fwd_tflops=(4 / 14) * flops / parts["fwd"] / 1e12 if parts.get("fwd") else None,
                bwd_tflops=(10 / 14) * flops / parts["bwd"] / 1e12 if parts.get("bwd") else None,
                affinity_cores=len(os.sched_getaffinity(0)))


def run_reference(a):
    _, rank, _ = rank_env()
    if rank != 0:          # the oracle runs once, on rank 0; the other ranks exit without work
        return
    from trainable_gated_block_b200 import inputs
    pc = inputs.workload(a.prefill)
    px = inputs.make_prefill(pc)
    per_step = 2
    for _ in range(a.warmup):
        _oracle_stripes(pc, px, 0.0, max_stripes=1)
    tot_f, tot_t, tot_n = 0, 0.0, 0
    for _ in range(a.steps):
        f, n, t = _oracle_stripes(pc, px, 1e9, max_stripes=per_step)
        tot_f, tot_t, tot_n = tot_f + f, tot_t + t, tot_n + n
    value = tot_f / tot_t / 1e12
    cores = _blas_threads()
    sample = (f"each step: fp64 oracle forward+backward of {per_step} 64-row stripes of the {pc.name} "
              f"workload (attended-tile flops); {tot_n} stripes in {tot_t:.1f} s")
    line = {
        "impl": "reference",
        "metric": "SAS gated block-sparse attn fwd+bwd TFLOPS & decode HBM GB/s vs roofline",
        "value": value, "unit": "TFLOPS", "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": tot_t / a.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{pc.name} select+fwd+bwd (oracle sample)"},
        "cpu_baseline": dict(value=value, unit="TFLOPS", cores=cores, kind="oracle", sample=sample),
        "e2e": dict(value=value, unit="TFLOPS", h2d_bytes_per_step=0, d2h_bytes_per_step=0),
    }
    print(json.dumps(line))


if __name__ == "__main__":
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
