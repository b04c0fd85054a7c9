"""The oracle against its pins, and the pins against planted oracle mistakes.

Every mutant below is a plausible slip in ``oracle/sas_oracle.py`` (a dropped
term, a wrong sign, index or operand, a misplaced scale). Each is planted in
a copy of the oracle's source on the CPU, and at least one pin must fail on
it; otherwise the pins would not be able to tell a wrong oracle from a right
one.
"""
import importlib.util
import inspect
import types

import pytest

from oracle import sas_oracle
from tests import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(sas_oracle)


MUTANTS = {
    "lse_over_selected_only": ("lse = logsumexp(row)\n", "lse = logsumexp(row[sel])\n"),
    "gate_sign_flipped": ("log_gate[b, h, r, slot] = row[j] - lse", "log_gate[b, h, r, slot] = lse - row[j]"),
    "tie_break_higher_index": ("np.lexsort((np.arange(nh), -s_row))", "np.lexsort((-np.arange(nh), -s_row))"),
    "causal_mask_off_by_one": ("np.where(u <= t, 0.0, NEG_INF)", "np.where(u < t + (t == 0), 0.0, NEG_INF)"),
    "current_block_gated": ("bias[:, rows] = np.where(u <= t, 0.0, NEG_INF)",
                            "bias[:, rows] = np.where(u <= t, (gates[0] if gates else 0.0), NEG_INF)"),
    "scale_applied_to_gate": ("L = sm_scale * (Qi @ Kh.T) + stripe_bias(i, S, sel, gates)",
                              "L = sm_scale * ((Qi @ Kh.T) + stripe_bias(i, S, sel, gates))"),
    "gqa_head_map_modulo": ("h = hq // G\n    sel, gates", "h = hq % k.shape[2]\n    sel, gates"),
    "jacobian_term_dropped": ("ds[b, h, i, :i] = -p * tot", "ds[b, h, i, :i] = 0.0 * p * tot"),
    "dk_missing_scale": ("dk[b, :, h, :] += sm_scale * (dS.T @ Qi)", "dk[b, :, h, :] += (dS.T @ Qi)"),
    "dP_wrong_operand": ("dP = dOi @ Vh.T", "dP = dOi @ Kh.T"),
    "gate_sum_wrong_axis": ("reshape(len(Qi), i, BLOCK).sum(axis=(0, 2))",
                            "reshape(len(Qi), i, BLOCK).sum(axis=(2, 0))[::-1]"),
    "Dr_dropped": ("dS = P * (dP - Dr)", "dS = P * dP"),
    "decode_current_block_short": ("bias[c * BLOCK:L] = 0.0", "bias[c * BLOCK:L - 1 + (L - 1 == c * BLOCK)] = 0.0"),
    "decode_history_includes_current": ("return (_i64(kv_len) - 1) // BLOCK", "return (_i64(kv_len) + BLOCK - 1) // BLOCK"),
    "prefill_history_includes_current": ("return np.arange(n_rows, dtype=np.int64)",
                                         "return np.arange(n_rows, dtype=np.int64) + 1"),
    "dq_missing_scale": ("dq[b, rs, hq, :] = sm_scale * (dS @ Kh)", "dq[b, rs, hq, :] = (dS @ Kh)"),
    "topk_lowest_scores": ("np.lexsort((np.arange(nh), -s_row))", "np.lexsort((np.arange(nh), s_row))"),
    "fwd_lse_missing_max": ("return P @ Vh, m[:, 0] + np.log(Z[:, 0]), P, L", "return P @ Vh, np.log(Z[:, 0]), P, L"),
    "jacobian_softmax_over_selected": ("p = np.exp(row - logsumexp(row))",
                                       "p = np.exp(row - logsumexp(row[sel])) * np.isin(np.arange(i), sel)"),
    "decode_gate_sign": ("bias[j * BLOCK:(j + 1) * BLOCK] = log_gate[n, h, slot]",
                         "bias[j * BLOCK:(j + 1) * BLOCK] = -log_gate[n, h, slot]"),
    "decode_page_offset": ("off = pos % BLOCK", "off = (pos + 1) % BLOCK"),
    "decode_lse_missing_max": ("lse[n, hq] = m + math.log(z)", "lse[n, hq] = math.log(z)"),
    "dv_half": ("dv[b, :, h, :] += P.T @ dOi", "dv[b, :, h, :] += 0.5 * (P.T @ dOi)"),
    "selection_left_in_score_order": ("return sorted(int(j) for j in order[:min(K, nh)])",
                                      "return [int(j) for j in order[:min(K, nh)]]"),
    "standin_sum_not_mean": ("qp = q.reshape(B, NQB, BLOCK, Hkv, G, D).mean(axis=(2, 4))",
                             "qp = q.reshape(B, NQB, BLOCK, Hkv, G, D).sum(axis=(2, 4))"),
    "standin_heads_interleaved": ("qp = q.reshape(B, NQB, BLOCK, Hkv, G, D).mean(axis=(2, 4))",
                                  "qp = q.reshape(B, NQB, BLOCK, G, Hkv, D).mean(axis=(2, 3))"),
    "standin_scale_d": ("s[b, h] = (qp[b, :, h, :] @ kp[b, :, h, :].T) / math.sqrt(D)",
                        "s[b, h] = (qp[b, :, h, :] @ kp[b, :, h, :].T) / D"),
    "partial_block_keys_dropped": ("bias[:, rows] = np.where(u <= t, 0.0, NEG_INF)",
                                   "bias[:, rows.start:rows.start + n - (n < BLOCK)] = np.where(u <= t, 0.0, NEG_INF)[:, :n - (n < BLOCK)]"),
    "varlen_kv_of_first_sequence": ("ob, lb = attn_fwd(q[None, rows], k[None, rows], v[None, rows],",
                                    "ob, lb = attn_fwd(q[None, rows], k[None, :L], v[None, :L],"),
    "varlen_selection_of_first_sequence": ("        ob, lb = attn_fwd(q[None, rows], k[None, rows], v[None, rows], idx[b:b + 1, :, :nb],\n"
                                           "                          cnt[b:b + 1, :, :nb], log_gate[b:b + 1, :, :nb], sm_scale)",
                                           "        ob, lb = attn_fwd(q[None, rows], k[None, rows], v[None, rows], idx[:1, :, :nb],\n"
                                           "                          cnt[:1, :, :nb], log_gate[:1, :, :nb], sm_scale)"),
    "varlen_bwd_dk_misplaced": ("dq[rows], dk[rows], dv[rows] = g[0][0], g[1][0], g[2][0]",
                                "dq[rows], dk[rows], dv[rows] = g[0][0], g[2][0], g[1][0]"),
    "varlen_ds_scores_of_first_sequence": ("cnt[b:b + 1, :, :nb], log_gate[b:b + 1, :, :nb], s[b:b + 1, :, :nb, :nb], sm_scale)",
                                           "cnt[b:b + 1, :, :nb], log_gate[b:b + 1, :, :nb], s[:1, :, :nb, :nb], sm_scale)"),
    "standin_decode_page_not_gathered": ("km = kc[pt[n, j], h].mean(axis=0)", "km = kc[j, h].mean(axis=0)"),
    "standin_decode_query_head_zero": ("qm = q[n, h * G:(h + 1) * G].mean(axis=0)", "qm = q[n, h * G]"),
    "standin_decode_history_includes_current": ("nh = int((kv_len[n] - 1) // BLOCK)\n        for h in range(Hkv):\n            qm",
                                                "nh = int((kv_len[n] + BLOCK - 1) // BLOCK)\n        for h in range(Hkv):\n            qm"),
    "standin_transposed": ("s[b, h] = (qp[b, :, h, :] @ kp[b, :, h, :].T) / math.sqrt(D)",
                           "s[b, h] = (kp[b, :, h, :] @ qp[b, :, h, :].T) / math.sqrt(D)"),
    "attended_tiles_without_current_block": ("return int((cnt + 1).sum()) * (Hq // Hkv)",
                                             "return int(cnt.sum()) * (Hq // Hkv)"),
}


def _mutant(src_from, src_to):
    src = inspect.getsource(sas_oracle)
    assert src.count(src_from) == 1, src_from
    mod = types.ModuleType("sas_oracle_mutant")
    exec(compile(src.replace(src_from, src_to), "sas_oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mod = _mutant(*MUTANTS[name])
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(mod)
        except Exception:          # an assertion, or a crash the slip causes
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name!r}"


def test_workload_scores_are_the_standin_definition():
    """The seeded 8k/32k workloads' scores are the oracle's stand-in scores plus the N(0,1)
    noise drawn fourth (after q, k, v) from the workload's generator, rounded to fp32 once."""
    import torch

    from trainable_gated_block_b200 import inputs
    cfg = inputs.PrefillConfig("standin-small", "bf16", 1, 512, 8, 2, 128, 4, "standin", seed=41)
    x = inputs.make_prefill(cfg, with_do=False)
    g = torch.Generator().manual_seed(41)
    q = inputs._randn((1, 512, 8, 128), g, torch.bfloat16)
    k = inputs._randn((1, 512, 2, 128), g, torch.bfloat16)
    inputs._randn((1, 512, 2, 128), g, torch.bfloat16)            # v
    noise = inputs._randn((1, 2, 8, 8), g, torch.float32)
    assert torch.equal(q, x["q"]) and torch.equal(k, x["k"])
    ref = sas_oracle.standin_scores(q, k, noise).astype("float32")
    assert (ref == x["s"].numpy()).all()
