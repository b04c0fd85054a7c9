"""Plain fp64 CPU oracle for SAS gated block-sparse causal attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product (the CUDA library ``libsas.so`` and its Python binding)
never calls it, and the two share no code: this file imports numpy only.

It is slow on purpose. Every step is the textbook definition, in fp64, with
the full masked logit matrix materialised 64 query rows at a time, a dense
softmax, and a backward pass differentiated by hand. Inputs arrive as the
exact fp32/bf16 values the GPU sees and are upcast to fp64 once.

Method (SAS review (paper.oopus.info), §2.1-§2.6; SAS abstract (fugumt.com)):

* §2.1: the context is cut into blocks of b = 64 tokens. The current block
  (the one holding the query) is always attended.
* §2.2: the selector scores every history block; the Top-K scores are kept.
* §2.4, eq. log g: each selected history block m gets the log-gate
  ``log g_m = s_m - LSE(s)``, the LSE taken over ALL history blocks; the
  current block has ``g_0 = 1`` (log-gate 0).
* §2.3, eq. o_SAS: ``o = softmax(q K_S^T + log g_S) V_S`` with the gate
  inside the softmax, in log form, over the selected set S.
* §2.6: the gradient of a block's gate is the sum of the logit gradients
  inside that block; it reaches the scores through the LSE Jacobian.

Readings taken where the pages are silent:

* the logits are ``sm_scale * q.k + log g``, sm_scale scaling q.k only;
* history of query block i = blocks 0..i-1; block 0 has no history, no gate;
* selection is per (batch, KV head, query block) and is shared by the GQA
  group; query head hq uses KV head ``hq // G``;
* Top-K order key (score descending, block index ascending), so the lower
  index wins a tie; -0.0 and +0.0 are equal scores; scores must be finite;
  with fewer than K history blocks all are selected;
* selected indices are reported ascending, padded with -1 (log-gate -inf);
* LSE of an empty history is -inf; all LSEs are natural logarithms;
* decode: the query sits at position ``kv_len-1``; its current block is
  ``c = (kv_len-1)//64`` holding tokens ``64c..kv_len-1``; its history is
  blocks ``0..c-1``.
* a prefill length S that is not a multiple of 64 ends in a partial block
  ``ceil(S/64)-1`` of ``S - 64*(ceil(S/64)-1)`` tokens: it is a query block
  like any other (its rows attend its own keys causally and its kept history
  blocks), and as a history block of no later query block it is never
  selected; the same rule as decode's partial current block.
* a batch of sequences of different lengths (packed along the token axis,
  sequence b holding tokens ``cu_seqlens[b]..cu_seqlens[b+1]-1``) is the
  method applied to each sequence on its own; the per-block tensors (scores,
  selection, ds) and the row LSE keep a padded ``[B, ..., max blocks]`` /
  ``[B, Hq, max length]`` layout whose entries past a sequence's end are
  padding.

Parity pins for every function are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64
NEG_INF = -np.inf


def _f64(x):
    """Upcast a numpy array or a CPU torch tensor (fp32 or bf16) to fp64 numpy."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _i64(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.asarray(x, dtype=np.int64)


# ----------------------------------------------------------------------------
# Selection and log-gates: SAS review §2.2 (Top-K over history blocks) and
# §2.4, eq. log g (log g_m = s_m - LSE over all history blocks).
# ----------------------------------------------------------------------------

def prefill_history(n_rows: int) -> np.ndarray:
    """History length (in blocks) of prefill query block i: blocks 0..i-1."""
    return np.arange(n_rows, dtype=np.int64)


def decode_history(kv_len) -> np.ndarray:
    """History length of a decode query at position kv_len-1: (kv_len-1)//64."""
    return (_i64(kv_len) - 1) // BLOCK


def topk_history(s_row, nh: int, K: int) -> list[int]:
    """Top-K history blocks of one row, by (score descending, index ascending).

    Returns the selected block indices in ascending order (SAS review §2.2).
    """
    s_row = _f64(s_row)[:nh]
    if not np.all(np.isfinite(s_row)):
        raise ValueError("selector scores must be finite")
    order = np.lexsort((np.arange(nh), -s_row))    # primary: -s, secondary: j
    return sorted(int(j) for j in order[:min(K, nh)])


def logsumexp(x) -> float:
    x = _f64(x)
    if x.size == 0:
        return -math.inf
    m = float(np.max(x))
    return m + math.log(float(np.sum(np.exp(x - m))))


def select(s, K: int, n_hist):
    """Top-K + log-gates for every row of a score tensor.

    s: [B, Hkv, R, ld] scores; row r of (b, h) reads ``s[b,h,r,0:n_hist]``.
    n_hist: int array broadcastable to [B, R] (prefill: r; decode: per b).
    Returns idx int32 [B,Hkv,R,K] (ascending, -1 padded), cnt int32
    [B,Hkv,R], log_gate fp64 [B,Hkv,R,K] (-inf padded), lse_s fp64 [B,Hkv,R].
    """
    s = _f64(s)
    B, H, R, _ = s.shape
    nh = np.broadcast_to(_i64(n_hist), (B, R))
    idx = np.full((B, H, R, K), -1, dtype=np.int32)
    cnt = np.zeros((B, H, R), dtype=np.int32)
    log_gate = np.full((B, H, R, K), NEG_INF)
    lse_s = np.full((B, H, R), NEG_INF)
    for b in range(B):
        for h in range(H):
            for r in range(R):
                n = int(nh[b, r])
                row = s[b, h, r, :n]
                sel = topk_history(row, n, K)
                lse = logsumexp(row)
                cnt[b, h, r] = len(sel)
                lse_s[b, h, r] = lse
                for slot, j in enumerate(sel):
                    idx[b, h, r, slot] = j
                    log_gate[b, h, r, slot] = row[j] - lse
    return idx, cnt, log_gate, lse_s


# ----------------------------------------------------------------------------
# Gated attention, forward: SAS review §2.3, eq. o_SAS, with the current block
# kept ungated (§2.4, g_0 = 1) under a causal mask.
# ----------------------------------------------------------------------------

def block_rows(i: int, S: int) -> slice:
    """Token rows of block i in a sequence of S tokens (the last block may be partial)."""
    return slice(i * BLOCK, min(S, (i + 1) * BLOCK))


def n_blocks(S: int) -> int:
    """Blocks of a sequence of S tokens, the last one possibly partial."""
    return (S + BLOCK - 1) // BLOCK


def stripe_bias(i: int, S: int, sel, gates) -> np.ndarray:
    """Masked bias of the query rows of block i over all S keys.

    0 on the causal part of the current block, the block's log-gate on every
    key of a selected history block, -inf everywhere else. Block i has 64
    rows, or fewer when it is the last, partial block of the sequence.
    """
    rows = block_rows(i, S)
    n = rows.stop - rows.start
    bias = np.full((n, S), NEG_INF)
    for j, lg in zip(sel, gates):
        assert 0 <= j < i
        bias[:, j * BLOCK:(j + 1) * BLOCK] = lg
    t = np.arange(n)[:, None]
    u = np.arange(n)[None, :]
    bias[:, rows] = np.where(u <= t, 0.0, NEG_INF)
    return bias


def _row_selection(idx, cnt, log_gate, b, h, i):
    c = int(cnt[b, h, i])
    return [int(j) for j in idx[b, h, i, :c]], [float(g) for g in log_gate[b, h, i, :c]]


def fwd_stripe(q, k, v, idx, cnt, log_gate, sm_scale, b, hq, i):
    """One stripe (the n <= 64 rows of block i): returns (o [n,D], lse [n], P [n,S], L [n,S])."""
    S = q.shape[1]
    G = q.shape[2] // k.shape[2]
    h = hq // G
    sel, gates = _row_selection(idx, cnt, log_gate, b, h, i)
    Qi = q[b, block_rows(i, S), hq, :]
    Kh = k[b, :, h, :]
    Vh = v[b, :, h, :]
    L = sm_scale * (Qi @ Kh.T) + stripe_bias(i, S, sel, gates)
    m = L.max(axis=1, keepdims=True)
    E = np.exp(L - m)
    Z = E.sum(axis=1, keepdims=True)
    P = E / Z
    return P @ Vh, m[:, 0] + np.log(Z[:, 0]), P, L


def attn_fwd(q, k, v, idx, cnt, log_gate, sm_scale, stripes=None):
    """Forward over all stripes (or the given (b, hq, i) stripes).

    q [B,S,Hq,D], k/v [B,S,Hkv,D]. Returns o fp64 [B,S,Hq,D] and lse fp64
    [B,Hq,S]; rows outside the requested stripes are NaN.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    idx, cnt, log_gate = _i64(idx), _i64(cnt), _f64(log_gate)
    B, S, Hq, D = q.shape
    o = np.full((B, S, Hq, D), np.nan)
    lse = np.full((B, Hq, S), np.nan)
    if stripes is None:
        stripes = [(b, hq, i) for b in range(B) for hq in range(Hq) for i in range(n_blocks(S))]
    for b, hq, i in stripes:
        oi, li, _, _ = fwd_stripe(q, k, v, idx, cnt, log_gate, sm_scale, b, hq, i)
        o[b, block_rows(i, S), hq, :] = oi
        lse[b, hq, block_rows(i, S)] = li
    return o, lse


# ----------------------------------------------------------------------------
# Backward by hand: SAS review §2.6 (gate gradient = sum of the logit gradients
# inside the block) and §2.4, eq. log g (its Jacobian with respect to s).
# ----------------------------------------------------------------------------

def attn_bwd(q, k, v, do, idx, cnt, log_gate, s, sm_scale, stripes=None):
    """Gradients of <o, dO> with respect to q, k, v and the scores s.

    Over all stripes by default. With ``stripes`` = a list of (b, hq, i),
    only those stripes contribute: dq and the gate sums are exact for them,
    and dk/dv of a key block are exact when every stripe that attends it is
    listed. Returns dq, dk, dv (fp64, input layouts), ds fp64 [B,Hkv,NQB,NQB]
    (zero on j >= i) and gsum fp64 [B,Hkv,NQB,NQB] (the per-block gate
    gradients dL/dlog g_ij, zero where j is not selected); NQB = ceil(S/64).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    idx, cnt, log_gate, s = _i64(idx), _i64(cnt), _f64(log_gate), _f64(s)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    NQB = n_blocks(S)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    gsum = np.zeros((B, Hkv, NQB, NQB))
    if stripes is None:
        stripes = [(b, hq, i) for b in range(B) for hq in range(Hq) for i in range(NQB)]
    rows_done = set()
    for b, hq, i in stripes:
        h = hq // G
        _, _, P, _ = fwd_stripe(q, k, v, idx, cnt, log_gate, sm_scale, b, hq, i)
        rs = block_rows(i, S)
        Qi, dOi = q[b, rs, hq, :], do[b, rs, hq, :]
        Kh, Vh = k[b, :, h, :], v[b, :, h, :]
        dv[b, :, h, :] += P.T @ dOi
        dP = dOi @ Vh.T
        Dr = np.sum(P * dP, axis=1, keepdims=True)
        dS = P * (dP - Dr)                       # gradient of the logits
        dq[b, rs, hq, :] = sm_scale * (dS @ Kh)
        dk[b, :, h, :] += sm_scale * (dS.T @ Qi)
        if i > 0:
            gsum[b, h, i, :i] += dS[:, :i * BLOCK].reshape(len(Qi), i, BLOCK).sum(axis=(0, 2))
        rows_done.add((b, h, i))
    ds = np.zeros((B, Hkv, NQB, NQB))
    for b, h, i in rows_done:
        if i == 0:
            continue
        sel = [int(j) for j in idx[b, h, i, :int(cnt[b, h, i])]]
        row = s[b, h, i, :i]
        p = np.exp(row - logsumexp(row))         # softmax(s_i) over all history
        tot = sum(gsum[b, h, i, m] for m in sel)
        ds[b, h, i, :i] = -p * tot
        for m in sel:
            ds[b, h, i, m] += gsum[b, h, i, m]
    return dq, dk, dv, ds, gsum


# ----------------------------------------------------------------------------
# Batches of sequences of different lengths, packed along the token axis: the
# method (SAS review §2.1-§2.6) applied to each sequence on its own.
# ----------------------------------------------------------------------------

def seq_bounds(cu_seqlens):
    """(start, length) of every sequence of a packed batch."""
    cu = _i64(cu_seqlens)
    return [(int(cu[b]), int(cu[b + 1] - cu[b])) for b in range(len(cu) - 1)]


def select_varlen(s, K: int, cu_seqlens):
    """select() per sequence: s [B, Hkv, R, ld] with R >= the most blocks of any
    sequence; row i of sequence b is a query block when i < ceil(len_b/64) and
    padding otherwise (cnt 0, idx -1, log-gate -inf, lse_s -inf)."""
    s = _f64(s)
    B, H, R, _ = s.shape
    idx = np.full((B, H, R, K), -1, dtype=np.int32)
    cnt = np.zeros((B, H, R), dtype=np.int32)
    log_gate = np.full((B, H, R, K), NEG_INF)
    lse_s = np.full((B, H, R), NEG_INF)
    for b, (_, L) in enumerate(seq_bounds(cu_seqlens)):
        nb = n_blocks(L)
        if nb == 0:
            continue
        out = select(s[b:b + 1, :, :nb], K, prefill_history(nb))
        idx[b, :, :nb], cnt[b, :, :nb], log_gate[b, :, :nb], lse_s[b, :, :nb] = (x[0] for x in out)
    return idx, cnt, log_gate, lse_s


def attn_fwd_varlen(q, k, v, cu_seqlens, idx, cnt, log_gate, sm_scale, max_seqlen: int, seqs=None):
    """attn_fwd() per sequence of a packed batch: q [T,Hq,D], k/v [T,Hkv,D].

    Returns o fp64 [T,Hq,D] and lse fp64 [B,Hq,max_seqlen]; entries past a
    sequence's length, and rows of sequences outside ``seqs``, are NaN.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    idx, cnt, log_gate = _i64(idx), _i64(cnt), _f64(log_gate)
    bounds = seq_bounds(cu_seqlens)
    o = np.full(q.shape, np.nan)
    lse = np.full((len(bounds), q.shape[1], max_seqlen), np.nan)
    for b, (st, L) in enumerate(bounds):
        if L == 0 or (seqs is not None and b not in seqs):
            continue
        nb = n_blocks(L)
        rows = slice(st, st + L)
        ob, lb = attn_fwd(q[None, rows], k[None, rows], v[None, rows], idx[b:b + 1, :, :nb],
                          cnt[b:b + 1, :, :nb], log_gate[b:b + 1, :, :nb], sm_scale)
        o[rows] = ob[0]
        lse[b, :, :L] = lb[0]
    return o, lse


def attn_bwd_varlen(q, k, v, do, cu_seqlens, idx, cnt, log_gate, s, sm_scale, seqs=None):
    """attn_bwd() per sequence of a packed batch. Returns dq, dk, dv ([T, H, D])
    and ds [B, Hkv, R, ld] (padding rows and sequences outside ``seqs`` zero)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    idx, cnt, log_gate, s = _i64(idx), _i64(cnt), _f64(log_gate), _f64(s)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    ds = np.zeros(s.shape)
    for b, (st, L) in enumerate(seq_bounds(cu_seqlens)):
        if L == 0 or (seqs is not None and b not in seqs):
            continue
        nb = n_blocks(L)
        rows = slice(st, st + L)
        g = attn_bwd(q[None, rows], k[None, rows], v[None, rows], do[None, rows], idx[b:b + 1, :, :nb],
                     cnt[b:b + 1, :, :nb], log_gate[b:b + 1, :, :nb], s[b:b + 1, :, :nb, :nb], sm_scale)
        dq[rows], dk[rows], dv[rows] = g[0][0], g[1][0], g[2][0]
        ds[b, :, :nb, :nb] = g[3][0]
    return dq, dk, dv, ds


# ----------------------------------------------------------------------------
# Paged decode: the same gated softmax for one query token per sequence, keys
# and values gathered through a page table of 64-token pages (SAS review §2.6:
# the serving side keeps the KV cache in pages).
# ----------------------------------------------------------------------------

def decode(q, k_cache, v_cache, page_table, kv_len, idx, cnt, log_gate, sm_scale, seqs=None):
    """q [N,Hq,D]; caches [P,Hkv,64,D]; selection [N,Hkv,K]. Returns o, lse.

    Rows of sequences outside ``seqs`` are NaN.
    """
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    pt, kv_len = _i64(page_table), _i64(kv_len)
    idx, cnt, log_gate = _i64(idx), _i64(cnt), _f64(log_gate)
    N, Hq, D = q.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    o = np.full((N, Hq, D), np.nan)
    lse = np.full((N, Hq), np.nan)
    for n in (range(N) if seqs is None else seqs):
        L = int(kv_len[n])
        pos = np.arange(L)
        page = pt[n, pos // BLOCK]
        off = pos % BLOCK
        c = (L - 1) // BLOCK
        for h in range(Hkv):
            Kn = kc[page, h, off, :]
            Vn = vc[page, h, off, :]
            bias = np.full(L, NEG_INF)
            bias[c * BLOCK:L] = 0.0
            for slot in range(int(cnt[n, h])):
                j = int(idx[n, h, slot])
                assert 0 <= j < c
                bias[j * BLOCK:(j + 1) * BLOCK] = log_gate[n, h, slot]
            for g in range(G):
                hq = h * G + g
                logits = sm_scale * (Kn @ q[n, hq]) + bias
                m = logits.max()
                e = np.exp(logits - m)
                z = e.sum()
                o[n, hq] = (e / z) @ Vn
                lse[n, hq] = m + math.log(z)
    return o, lse


# ----------------------------------------------------------------------------
# Stand-in selector scores: the step before select. The pages' selector
# (AttnGate, SAS review §2.2) needs trained weights, so its scores are stood in
# for by pooled attention logits: the mean of q over the 64 rows of block i and
# the G query heads of KV head h, dotted with the mean of k[h] over the 64 rows
# of block j, over sqrt(D), plus a given noise term (the random part is an
# input, drawn by the caller).
# ----------------------------------------------------------------------------

def standin_scores(q, k, noise):
    """s[b, h, i, j] = mean_{64 rows of block i, G heads of h}(q) . mean_{64 rows of block j}(k[:, :, h]) / sqrt(D)
    + noise[b, h, i, j], in fp64. q [B,S,Hq,D], k [B,S,Hkv,D], noise [B,Hkv,NQB,NQB]; every
    (i, j) is produced (select reads only j < i)."""
    q, k, noise = _f64(q), _f64(k), _f64(noise)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    NQB = S // BLOCK
    qp = q.reshape(B, NQB, BLOCK, Hkv, G, D).mean(axis=(2, 4))      # [B, NQB, Hkv, D]
    kp = k.reshape(B, NQB, BLOCK, Hkv, D).mean(axis=2)              # [B, NQB, Hkv, D]
    s = np.zeros((B, Hkv, NQB, NQB))
    for b in range(B):
        for h in range(Hkv):
            s[b, h] = (qp[b, :, h, :] @ kp[b, :, h, :].T) / math.sqrt(D)
    return s + noise


def standin_scores_decode(q, k_cache, page_table, kv_len, noise):
    """Stand-in scores of decode queries: s[n, h, j] = mean over the G query heads of KV
    head h of q[n] . mean over the 64 rows of page page_table[n, j] of k_cache[:, h] /
    sqrt(D) + noise[n, h, j], in fp64, for the history blocks j < (kv_len[n]-1)//64 (the
    other entries are NaN). q [N,Hq,D], k_cache [P,Hkv,64,D], noise [N,Hkv,ld]."""
    q, kc, noise = _f64(q), _f64(k_cache), _f64(noise)
    pt, kv_len = _i64(page_table), _i64(kv_len)
    N, Hq, D = q.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    s = np.full(noise.shape, np.nan)
    for n in range(N):
        nh = int((kv_len[n] - 1) // BLOCK)
        for h in range(Hkv):
            qm = q[n, h * G:(h + 1) * G].mean(axis=0)
            for j in range(nh):
                km = kc[pt[n, j], h].mean(axis=0)
                s[n, h, j] = float(qm @ km) / math.sqrt(D) + noise[n, h, j]
    return s


# ----------------------------------------------------------------------------
# Work counts used to express throughput (not part of the method).
# ----------------------------------------------------------------------------

def attended_tiles(cnt, Hq: int, Hkv: int) -> int:
    """64x64 tiles attended over all query heads: (selected + current) blocks."""
    cnt = _i64(cnt)
    return int((cnt + 1).sum()) * (Hq // Hkv)
