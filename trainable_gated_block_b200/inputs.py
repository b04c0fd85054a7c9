"""Seeded synthetic inputs for SAS gated block-sparse attention.

This module only draws random tensors. It holds none of the method's
arithmetic (no Top-K, no gates, no attention): the oracle and the CUDA path
both start from the tensors it returns, so both see identical bits.

Workloads (one per named shape; sizes follow the Qwen3 attention layers the
SAS pages train, with the pages' token budgets 1024/2048/512 at b = 64):

* ``tiny-fp32``         fp32, B=1, S=512, 2 query heads on 1 KV head, D=64, K=2
* ``qwen3-4b-8k``       bf16, B=1, S=8192, 32/8 heads, D=128, K=16
* ``qwen3-8b-32k``      bf16, B=1, S=32768, 32/8 heads, D=128, K=32
* ``qwen3-14b-2x32k``   bf16, B=2, S=32768, 40/8 heads, D=128, K=8
* ``decode-64seq``      bf16 paged decode, 64 sequences, 32/8 heads, D=128, K=32

Draw order from one ``torch.Generator`` seeded with the workload's seed:
prefill q, k, v, then the score noise (or the scores), then dO; decode q,
history lengths, page permutation, k cache, v cache, scores.

The Qwen3-shaped prefill workloads (8k and 32k) take their selector scores
from a block-pooled stand-in for the selector ``s = R_theta(q, {K_Bm})``
(SAS review (paper.oopus.info), §2.2): the mean of the query block's queries
over its GQA head group, dotted with the mean of the key block's keys, over
sqrt(D), plus N(0,1) noise. The real selector (AttnGate) needs trained
weights that are not available, so this is input generation, not the method.
It is computed in fp64 from the rounded q/k and rounded to fp32 once.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

BLOCK = 64


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    dtype: str          # "f32" or "bf16": the dtype of q, k, v, o, dO
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    K: int              # Top-K budget in history blocks
    scores: str         # "normal" (i.i.d. N(0, score_std)) or "standin"
    score_std: float = 1.0
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def NQB(self) -> int:
        return (self.S + BLOCK - 1) // BLOCK

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    N: int              # sequences, one query token each
    Hq: int
    Hkv: int
    D: int
    K: int
    min_hist: int = 128     # history length in blocks, drawn U{min_hist..max_hist}
    max_hist: int = 1024
    partial: bool = False   # False: current block holds 1 token; True: U{1..64}
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS = {
    "tiny-fp32": PrefillConfig("tiny-fp32", "f32", 1, 512, 2, 1, 64, 2, "normal", 1.0, seed=1),
    "qwen3-4b-8k": PrefillConfig("qwen3-4b-8k", "bf16", 1, 8192, 32, 8, 128, 16, "standin", seed=2),
    "qwen3-8b-32k": PrefillConfig("qwen3-8b-32k", "bf16", 1, 32768, 32, 8, 128, 32, "standin", seed=3),
    "qwen3-14b-2x32k": PrefillConfig("qwen3-14b-2x32k", "bf16", 2, 32768, 40, 8, 128, 8, "normal", 2.0, seed=4),
    "decode-64seq": DecodeConfig("decode-64seq", 64, 32, 8, 128, 32, seed=5),
}


def workload(name: str, **overrides):
    cfg = WORKLOADS[name]
    return replace(cfg, **overrides) if overrides else cfg


def _randn(shape, g, dtype, chunk_elems=1 << 26):
    """N(0,1) draws in fp32, rounded once (RNE) to ``dtype``; chunked for big tensors."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=dtype)
    for lo in range(0, n, chunk_elems):
        hi = min(n, lo + chunk_elems)
        out[lo:hi] = torch.randn(hi - lo, generator=g, dtype=torch.float32).to(dtype)
    return out.view(shape)


def make_prefill(cfg: PrefillConfig, seed: int | None = None, with_do: bool = True):
    """Return a dict of CPU tensors: q, k, v ([B,S,H,D]), s ([B,Hkv,NQB,NQB] fp32), do.

    S need not be a multiple of 64 (NQB = ceil(S/64)) except for stand-in scores."""
    assert cfg.Hq % cfg.Hkv == 0 and (cfg.scores != "standin" or cfg.S % BLOCK == 0)
    g = torch.Generator().manual_seed(cfg.seed if seed is None else seed)
    dt = cfg.torch_dtype
    B, S, Hq, Hkv, D, NQB = cfg.B, cfg.S, cfg.Hq, cfg.Hkv, cfg.D, cfg.NQB
    q = _randn((B, S, Hq, D), g, dt)
    k = _randn((B, S, Hkv, D), g, dt)
    v = _randn((B, S, Hkv, D), g, dt)
    noise = _randn((B, Hkv, NQB, NQB), g, torch.float32)
    if cfg.scores == "normal":
        s = (noise.double() * cfg.score_std).float()
    elif cfg.scores == "standin":
        qp = q.double().view(B, NQB, BLOCK, Hkv, cfg.G, D).mean(dim=(2, 4))   # [B,NQB,Hkv,D]
        kp = k.double().view(B, NQB, BLOCK, Hkv, D).mean(dim=2)               # [B,NQB,Hkv,D]
        s = (torch.einsum("bihd,bjhd->bhij", qp, kp) / math.sqrt(D) + noise.double()).float()
    else:
        raise ValueError(cfg.scores)
    out = dict(q=q, k=k, v=v, s=s.contiguous())
    if cfg.scores == "standin":
        out["noise"] = noise            # the random part of the stand-in scores
    if with_do:
        out["do"] = _randn((B, S, Hq, D), g, dt)
    return out


def make_varlen(lengths, Hq: int, Hkv: int, D: int, dtype: str = "bf16", score_std: float = 1.0,
                seed: int = 0):
    """A packed batch of sequences of the given lengths (CPU tensors).

    Returns q, do [T,Hq,D], k, v [T,Hkv,D] (T = sum of lengths), cu_seqlens int32
    [B+1], max_seqlen, and scores s [B,Hkv,R,R] fp32 ~ N(0, score_std), R = the
    blocks of the longest sequence. Draw order: q, k, v, scores, dO.
    """
    g = torch.Generator().manual_seed(seed)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    T = int(sum(lengths))
    B = len(lengths)
    max_seqlen = max(lengths)
    R = (max_seqlen + BLOCK - 1) // BLOCK
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    q = _randn((T, Hq, D), g, dt)
    k = _randn((T, Hkv, D), g, dt)
    v = _randn((T, Hkv, D), g, dt)
    s = (_randn((B, Hkv, R, R), g, torch.float32).double() * score_std).float()
    do = _randn((T, Hq, D), g, dt)
    return dict(q=q, k=k, v=v, s=s.contiguous(), do=do, cu_seqlens=cu, max_seqlen=max_seqlen)


def make_decode(cfg: DecodeConfig, seed: int | None = None):
    """Paged-KV decode inputs (CPU tensors).

    Sequence n holds ``L_n = 64*U{min_hist..max_hist}`` cached tokens plus the
    current block (1 token, or U{1..64} with ``partial``), so
    ``kv_len = L_n + c_n``. Its ``ceil(kv_len/64)`` pages are scattered over
    the cache by one seeded permutation of all pages.
    Returns q [N,Hq,D], k_cache/v_cache [P,Hkv,64,D], page_table [N,max_pages]
    int32 (unused slots 0), kv_len [N] int32, s [N,Hkv,max_hist] fp32.
    """
    g = torch.Generator().manual_seed(cfg.seed if seed is None else seed)
    N, Hq, Hkv, D = cfg.N, cfg.Hq, cfg.Hkv, cfg.D
    q = _randn((N, Hq, D), g, torch.bfloat16)
    hist = torch.randint(cfg.min_hist, cfg.max_hist + 1, (N,), generator=g)
    if cfg.partial:
        cur = torch.randint(1, BLOCK + 1, (N,), generator=g)
    else:
        cur = torch.ones(N, dtype=torch.int64)
    kv_len = (hist * BLOCK + cur).to(torch.int32)
    pages = (kv_len.to(torch.int64) + BLOCK - 1) // BLOCK
    total = int(pages.sum())
    max_pages = cfg.max_hist + 1
    perm = torch.randperm(total, generator=g).to(torch.int32)
    page_table = torch.zeros((N, max_pages), dtype=torch.int32)
    off = 0
    for n in range(N):
        p = int(pages[n])
        page_table[n, :p] = perm[off:off + p]
        off += p
    k_cache = _randn((total, Hkv, BLOCK, D), g, torch.bfloat16)
    v_cache = _randn((total, Hkv, BLOCK, D), g, torch.bfloat16)
    s = _randn((N, Hkv, cfg.max_hist), g, torch.float32)
    return dict(q=q, k_cache=k_cache, v_cache=v_cache, page_table=page_table,
                kv_len=kv_len, s=s)


def make_decode_device(N: int, ctx: int, Hq: int, Hkv: int, D: int, seed: int, device):
    """Decode inputs drawn on the device, for timing studies whose caches are too large to
    draw on the host (batch 8 at 512K holds 17 GB of pages). Every sequence holds ``ctx``
    cached tokens plus one new token (kv_len = ctx + 1); its ctx/64 + 1 pages are scattered
    by one seeded permutation of all pages. Scores s [N, Hkv, ctx/64] ~ N(0,1)."""
    g = torch.Generator(device=device).manual_seed(seed)
    pages = ctx // BLOCK + 1
    total = N * pages
    page_table = torch.randperm(total, generator=g, device=device).to(torch.int32).view(N, pages).contiguous()
    kv_len = torch.full((N,), ctx + 1, dtype=torch.int32, device=device)
    q = torch.randn((N, Hq, D), generator=g, device=device).to(torch.bfloat16)
    k_cache = torch.randn((total, Hkv, BLOCK, D), generator=g, device=device, dtype=torch.bfloat16)
    v_cache = torch.randn((total, Hkv, BLOCK, D), generator=g, device=device, dtype=torch.bfloat16)
    s = torch.randn((N, Hkv, ctx // BLOCK), generator=g, device=device)
    return dict(q=q, k_cache=k_cache, v_cache=v_cache, page_table=page_table, kv_len=kv_len, s=s)
