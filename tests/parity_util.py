"""Comparison helpers for the GPU parity tests.

Tolerances (fp16/bf16 outputs with fp32 accumulation against the fp64 oracle):
  out: |gpu - ref| <= 2e-3 + 1e-2 * |ref| element by element
  lse: |gpu - ref| <= 1e-3 (natural log); -inf must match -inf exactly.
"""
from __future__ import annotations

import numpy as np
import torch

OUT_ATOL, OUT_RTOL, LSE_ATOL = 2e-3, 1e-2, 1e-3

BIAS_CODE = {"none": 0, "causal": 1, "blockdiag": 2, "blockdiag_causal": 3}


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def assert_out_close(gpu, ref, what=""):
    g, r = to_np(gpu), to_np(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - r)
    bad = err > OUT_ATOL + OUT_RTOL * np.abs(r)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; max abs err "
            f"{err.max():.3e}; first at {idx.tolist()}: gpu {g[tuple(idx[0])]} ref {r[tuple(idx[0])]}")


def assert_lse_close(gpu, ref, what=""):
    g, r = to_np(gpu), to_np(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    ninf_r, ninf_g = np.isneginf(r), np.isneginf(g)
    assert (ninf_r == ninf_g).all(), f"{what}: -inf pattern differs ({ninf_r.sum()} vs {ninf_g.sum()})"
    fin = ~ninf_r
    assert np.isfinite(g[fin]).all(), f"{what}: non-finite lse"
    err = np.abs(g[fin] - r[fin])
    if err.size and err.max() > LSE_ATOL:
        raise AssertionError(f"{what}: lse max abs err {err.max():.3e} ({(err > LSE_ATOL).sum()} bad)")


def prefill_oracle_code(bias: str) -> int:
    return BIAS_CODE[bias]
