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


# ---------------------------------------------------------------------------
# Guard bands: an output tensor is a view into the middle of a larger buffer
# whose ends hold a sentinel bit pattern; a kernel that writes past either end
# of its output changes a band.  Checked after every GPU call of the parity
# tests (the stand-in for a memory checker).
# ---------------------------------------------------------------------------
_INT_VIEW = {torch.float16: torch.int16, torch.bfloat16: torch.int16, torch.float32: torch.int32,
             torch.uint8: torch.uint8}
_SENTINEL = {torch.int16: 0x7E5A, torch.int32: 0x7FC0DEAD, torch.uint8: 0xA5}
BAND_BYTES = 8192  # a multiple of 256: the view keeps the allocation's alignment


class Guarded:
    """A tensor of `shape` with sentinel-filled bands before and after it."""

    def __init__(self, shape, dtype, device, fill=None):
        n = 1
        for s in shape:
            n *= int(s)
        esz = torch.empty((), dtype=dtype).element_size()
        self.band = BAND_BYTES // esz
        self.n = n
        self.buf = torch.empty(n + 2 * self.band, dtype=dtype, device=device)
        ity = _INT_VIEW[dtype]
        s = _SENTINEL[ity]
        if ity == torch.int16 and s >= 1 << 15:
            s -= 1 << 16
        if ity == torch.int32 and s >= 1 << 31:
            s -= 1 << 32
        self.buf.view(ity).fill_(s)
        self._bits = s
        self._ity = ity
        self.t = self.buf[self.band:self.band + n].view(*shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what=""):
        bits = self.buf.view(self._ity)
        lo, hi = bits[:self.band], bits[self.band + self.n:]
        assert bool((lo == self._bits).all()), f"{what}: write before the start of the output"
        assert bool((hi == self._bits).all()), f"{what}: write past the end of the output"


def guarded_like(t: torch.Tensor, fill=None) -> Guarded:
    return Guarded(tuple(t.shape), t.dtype, t.device, fill)
