"""Helpers for comparing the CUDA path against the fp64 oracle.

Tolerances (what the tests assert):
* Top-K indices and counts: bit-exact.
* fp32 path: max-abs <= 1e-5 on o, lse, log_gate, lse_s, dq, dk, dv, ds.
* bf16 path: outputs o max-abs <= 1e-2 against the fp64 oracle, except
  where the bf16 output format itself cannot get that close: an output of
  magnitude >= 4 has a bf16 spacing of 2^-5, so rounding alone can move it
  by 2^-6 = 0.0156. There the test also requires the GPU value to be within
  1e-2 of the oracle value rounded to bf16 (RNE), and counts such elements.
  lse max-abs <= 1e-2. Gradients dq, dk, dv, ds: relative L2 <= 1e-2; where the
  exact gradient is identically zero, max-abs <= 1e-5 (rounding noise only).
"""
from __future__ import annotations

import numpy as np
import torch

FP32_TOL = 1e-5
BF16_OUT_TOL = 1e-2
BF16_GRAD_REL_L2 = 1e-2

# Every bf16 output comparison of the session: (what, elements, max_abs,
# max_abs against the oracle rounded to bf16, elements that pass only through
# the output-rounding exemption). Printed at the end of the run by conftest.py.
OUT_LOG: list[tuple[str, int, float, float, int]] = []


def np64(t):
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy().astype(np.float64)


def bf16_round(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def max_abs(a, b):
    a, b = np64(a), np64(b)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))


def rel_l2(a, b):
    a, b = np64(a), np64(b)
    den = float(np.linalg.norm(b.ravel()))
    return float(np.linalg.norm((a - b).ravel())) / max(den, 1e-30)


def check_out(gpu, ref, dtype: str, what: str):
    """Assert output parity; returns a dict of the measured errors."""
    g, r = np64(gpu), np64(ref)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU values"
    err = np.abs(g - r)
    if dtype == "f32":
        m = float(err.max(initial=0.0))
        assert m <= FP32_TOL, f"{what}: fp32 max-abs {m:.3e} > {FP32_TOL}"
        return dict(max_abs=m)
    rq = bf16_round(r)
    errq = np.abs(g - rq)
    over = err > BF16_OUT_TOL
    quant_only = over & (np.abs(r) >= 4.0) & (errq <= BF16_OUT_TOL)
    bad = over & ~quant_only
    assert not np.any(bad), (f"{what}: bf16 max-abs {err.max():.3e} > {BF16_OUT_TOL} "
                             f"at {int(bad.sum())} elements not explained by output rounding")
    res = dict(max_abs=float(err.max(initial=0.0)), max_abs_vs_rounded=float(errq.max(initial=0.0)),
               quantization_only=int(quant_only.sum()))
    OUT_LOG.append((what, int(err.size), res["max_abs"], res["max_abs_vs_rounded"], res["quantization_only"]))
    return res


def check_grad(gpu, ref, dtype: str, what: str):
    g, r = np64(gpu), np64(ref)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU values"
    if dtype == "f32":
        m = max_abs(g, r)
        assert m <= FP32_TOL, f"{what}: fp32 max-abs {m:.3e} > {FP32_TOL}"
        return dict(max_abs=m)
    if float(np.linalg.norm(r.ravel())) == 0.0:
        # the exact gradient is zero (e.g. a lone token attending only itself: P = 1 and
        # dP - Dr = 0): a relative error is undefined, so only rounding noise at the fp32
        # level is allowed
        m = float(np.abs(g).max(initial=0.0))
        assert m <= FP32_TOL, f"{what}: exact gradient is zero, GPU max-abs {m:.3e} > {FP32_TOL}"
        return dict(max_abs=m)
    e = rel_l2(g, r)
    assert e <= BF16_GRAD_REL_L2, f"{what}: bf16 rel-L2 {e:.3e} > {BF16_GRAD_REL_L2}"
    return dict(rel_l2=e)
