"""Parity of the backward kernels (mea_bwd, through the C ABI) with the fp64
oracle's gradients on the same seeded inputs and upstream gradient.

Tolerance (derived, gradients only): the GPU forms D_i = <dO_i, O_i> from the
forward's fp16/bf16 output O, whose rounding (relative 2^-11 / 2^-8) enters every
dS_ij = p_ij (dP_ij - D_i) of the row; P and dS are carried with >= 11 (fp16) or
~16 (bf16 hi+lo) significant bits and accumulated in fp32.  Elementwise:
    |g - ref| <= rtol * |ref| + atol * max|ref|,  rtol = 2e-2,
    atol = 4e-3 (fp16) / 1e-2 (bf16)  (per tensor: dq, dk, dv)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import BIAS_CODE, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def mea():
    import memory_efficient_exact_mea_b200 as m

    return m


def _assert_grad(g, ref, dtype, what):
    g, r = to_np(g), to_np(ref)
    assert np.isfinite(g).all(), f"{what}: non-finite"
    scale = np.abs(r).max() + 1e-30
    atol = (4e-3 if dtype == "f16" else 1e-2) * scale
    err = np.abs(g - r)
    bad = err > atol + 2e-2 * np.abs(r)
    assert not bad.any(), (f"{what}: {bad.sum()}/{bad.size} out of tolerance, max err "
                           f"{err.max():.3e} (scale {scale:.3e})")


def _check(mea, p: synth.Prefill):
    g = synth.generator(p.seed + 17)
    dout = synth.randn(tuple(p.q.shape), p.dtype, g)
    kw = {}
    if p.bias.startswith("blockdiag"):
        kw = dict(seqstart_q=p.seqstart_q.to(DEV), seqstart_k=p.seqstart_k.to(DEV))
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    out, lse = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=p.alibi, **kw)
    dq, dk, dv = mea.mea_bwd(q, k, v, out, dout.to(DEV), lse, bias=p.bias, scale=p.scale,
                             alibi=p.alibi, **kw)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    rq, rk, rv = oracle.get().attention_bwd(p.q, p.k, p.v, dout, bias=BIAS_CODE[p.bias],
                                            scale=p.scale, alibi=p.alibi,
                                            seqstart_q=p.seqstart_q, seqstart_k=p.seqstart_k)
    _assert_grad(dq, rq, p.dtype, f"{p.name} dq")
    _assert_grad(dk, rk, p.dtype, f"{p.name} dk")
    _assert_grad(dv, rv, p.dtype, f"{p.name} dv")


@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16"), (128, "f16"), (64, "bf16")])
@pytest.mark.parametrize("bias", ["none", "causal"])
def test_bwd_dense(mea, K, dtype, bias):
    p = synth.make_prefill(f"bwd_{bias}_{K}_{dtype}", 2, 200, 200, 4, 4, K, dtype, bias,
                           seed=200 + K)
    _check(mea, p)


@pytest.mark.parametrize("M,N", [(64, 64), (130, 70), (70, 130), (1, 5)])
def test_bwd_rectangular_causal(mea, M, N):
    p = synth.make_prefill(f"bwd_rect_{M}x{N}", 1, M, N, 2, 2, 64, "f16", "causal", seed=210 + M)
    _check(mea, p)


@pytest.mark.parametrize("alibi", [False, True])
def test_bwd_gqa(mea, alibi):
    p = synth.make_prefill(f"bwd_gqa_a{alibi}", 2, 256, 256, 8, 2, 128, "bf16", "causal",
                           alibi=alibi, seed=220)
    _check(mea, p)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_varlen(mea, causal):
    p = synth.make_varlen(f"bwd_varlen_c{causal}", [1, 63, 64, 65, 200, 0, 130], 4, 2, 128, "bf16",
                          causal, seed=230, alibi=causal)
    _check(mea, p)


@pytest.mark.parametrize("case", ["noncausal_b8_h16_m2048_k64_f16", "gqa_alibi_causal_b4_m4096"])
def test_bwd_full_size_properties(mea, case):
    """The benchmarked backward workloads, at full size, through properties that
    hold for every row: its weights sum to one, so per (batch, kv head) the keys'
    dv sum to the rows' dout summed over the head group; each row of dS sums to
    zero, so the keys' dk sum to zero.  Tolerance: the 16-bit rounding of each
    gradient element (relative 2^-9 bf16, 2^-12 fp16), against the sum of
    magnitudes."""
    p = synth.noncausal_sweep(2048) if case.startswith("noncausal") else synth.gqa_alibi_causal()
    dout = synth.randn(tuple(p.q.shape), p.dtype, synth.generator(p.seed + 17)).to(DEV)
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    out, lse = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=p.alibi)
    dq, dk, dv = mea.mea_bwd(q, k, v, out, dout, lse, bias=p.bias, scale=p.scale, alibi=p.alibi)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    for g in (dq, dk, dv):
        assert torch.isfinite(g).all()
    G = p.Hq // p.Hkv
    rel = 4e-3 if p.dtype == "bf16" else 5e-4
    sdv = dv.double().sum(dim=1)
    sdo = dout.double().view(p.B, p.M, p.Hkv, G, p.K).sum(dim=(1, 3))
    mag = dv.double().abs().sum(dim=1) + dout.double().abs().view(p.B, p.M, p.Hkv, G, p.K).sum(dim=(1, 3))
    assert ((sdv - sdo).abs() <= rel * mag + 1e-6).all(), (sdv - sdo).abs().max().item()
    sdk = dk.double().sum(dim=1)
    assert (sdk.abs() <= rel * dk.double().abs().sum(dim=1) + 1e-6).all(), sdk.abs().max().item()
