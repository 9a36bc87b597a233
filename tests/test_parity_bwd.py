"""Parity of the backward kernels (mea_bwd, through the C ABI) with the fp64
oracle's gradients on the same seeded inputs and upstream gradient.

Tolerance (gradients only).  Elementwise, per tensor (dq, dk, dv):
    |g - ref| <= rtol * |ref| + atol * max|ref|,  rtol = 2e-2,
    atol = 1e-3 (fp16) / 8e-3 (bf16).
Where the error comes from: the GPU forms D_i = <dO_i, O_i> from the forward's
16-bit output O, and P^T and dS^T enter the dV, dK and dQ products as single
16-bit values (relative rounding 2^-12 for fp16, 2^-9 for bf16), accumulated in
fp32; every gradient element sums many such terms, whose rounding errors mostly
cancel.  The largest atol any case here needed, measured on the GPU against the
oracle (every case of this file, the rescale file's backward and two groups of
each full-size workload), was 2.7e-4 (fp16) and 4.5e-3 (bf16, keys ramped 1 ->
16); the bounds above keep a margin of about 4x and 1.8x over those."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import BIAS_CODE, Guarded, to_np

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
    atol = (1e-3 if dtype == "f16" else 8e-3) * scale
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
    # gradients and the workspace between guard bands
    gq, gk, gv = (Guarded(tuple(t.shape), t.dtype, DEV, fill=float("nan")) for t in (q, k, v))
    B, M, Hq, K = q.shape
    gw = Guarded((max(1, mea.lib.mea_bwd_workspace_size(B, M, Hq, K)),), torch.uint8, DEV)
    dq, dk, dv = mea.mea_bwd(q, k, v, out, dout.to(DEV), lse, bias=p.bias, scale=p.scale,
                             alibi=p.alibi, dq=gq.t, dk=gk.t, dv=gv.t, workspace=gw.t, **kw)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    for g, nm in ((gq, "dq"), (gk, "dk"), (gv, "dv"), (gw, "workspace")):
        g.check(f"{p.name} {nm}")
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


@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16")])
@pytest.mark.parametrize("M,N", [(64, 64), (130, 70), (70, 130), (1, 5), (97, 300)])
def test_bwd_rectangular_causal(mea, M, N, K, dtype):
    """Row counts that end inside a 32-query half step (K = 128 stages dQ per half)
    and inside a 128-key block."""
    p = synth.make_prefill(f"bwd_rect_{M}x{N}_{K}", 1, M, N, 2, 2, K, dtype, "causal",
                           seed=210 + M)
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


def oracle_bwd_group(p: synth.Prefill, dout, b: int, g: int, chunk: int = 128):
    """The oracle's gradients for batch b and kv head g of a full-size problem
    (M = N): dq of the group's query heads (all rows) and dk, dv of kv head g.

    The work is cut into chunks of query rows run on host threads (ctypes drops
    the GIL): the forward treats rows independently, so a chunk's dq rows are
    its own, and dk, dv are the sums of the chunks' contributions.  Under the
    causal mask a chunk of rows [r0, r1) takes keys [0, r1): with the
    bottom-right alignment its row i' then sits at position i' + r0, the row's
    own position, which fixes both the mask and the ALiBi distances."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    G = p.Hq // p.Hkv
    causal = p.bias == "causal"
    assert p.M == p.N and p.bias in ("none", "causal") and not (p.alibi and not causal)
    orc = oracle.get()
    slopes = orc.alibi_slopes(p.Hq)[g * G:(g + 1) * G] if p.alibi else None
    qs = p.q[b:b + 1, :, g * G:(g + 1) * G].contiguous()
    ks = p.k[b:b + 1, :, g:g + 1].contiguous()
    vs = p.v[b:b + 1, :, g:g + 1].contiguous()
    ds = dout[b:b + 1, :, g * G:(g + 1) * G].contiguous()

    def job(r0):
        r1 = min(p.M, r0 + chunk)
        n = r1 if causal else p.N
        return r0, r1, orc.attention_bwd(qs[:, r0:r1], ks[:, :n], vs[:, :n], ds[:, r0:r1],
                                         bias=BIAS_CODE[p.bias], scale=p.scale, alibi=slopes)

    dq = np.zeros((p.M, G, p.K))
    dk = np.zeros((p.N, p.K))
    dv = np.zeros((p.N, p.K))
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        for r0, r1, (cq, ck, cv) in ex.map(job, range(0, p.M, chunk)):
            dq[r0:r1] = cq[0]
            dk[:ck.shape[1]] += ck[0, :, 0]
            dv[:cv.shape[1]] += cv[0, :, 0]
    return dq, dk, dv


@pytest.mark.parametrize("case", ["noncausal_b8_h16_m2048_k64_f16", "gqa_alibi_causal_b4_m4096"])
def test_bwd_full_size_elementwise(mea, case):
    """The benchmarked backward workloads at full size, through the same launch
    the bench times, compared element by element with the oracle on two
    (batch, kv head) groups: dq of every row of the group's query heads, dk and
    dv of every key of its kv head."""
    p = synth.noncausal_sweep(2048) if case.startswith("noncausal") else synth.gqa_alibi_causal()
    dout = synth.randn(tuple(p.q.shape), p.dtype, synth.generator(p.seed + 17))
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    out, lse = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=p.alibi)
    dq, dk, dv = mea.mea_bwd(q, k, v, out, dout.to(DEV), lse, bias=p.bias, scale=p.scale,
                             alibi=p.alibi)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    G = p.Hq // p.Hkv
    for b, g in ((0, 0), (p.B - 1, p.Hkv - 1)):
        rq, rk, rv = oracle_bwd_group(p, dout, b, g)
        _assert_grad(dq[b, :, g * G:(g + 1) * G].cpu(), rq, p.dtype, f"{case} b={b} g={g} dq")
        _assert_grad(dk[b, :, g].cpu(), rk, p.dtype, f"{case} b={b} g={g} dk")
        _assert_grad(dv[b, :, g].cpu(), rv, p.dtype, f"{case} b={b} g={g} dv")


def test_bwd_stages_one_by_one_equal_one_call(mea):
    """mea_bwd_stages: the preparation, main and dq stages run one by one on the
    same workspace give the gradients of one full call: dk, dv bit-identical
    (each key block accumulates on one CTA), dq within one unit in the last place
    (its fp32 accumulator is summed across key blocks by L2 reductions, in an
    order that varies from run to run)."""
    p = synth.make_prefill("bwd_stages", 2, 300, 260, 8, 2, 128, "bf16", "causal", alibi=True,
                           seed=240)
    dout = synth.randn(tuple(p.q.shape), p.dtype, synth.generator(p.seed + 17)).to(DEV)
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    out, lse = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=True)
    full = mea.mea_bwd(q, k, v, out, dout, lse, bias=p.bias, scale=p.scale, alibi=True)
    B, M, Hq, K = q.shape
    ws = torch.empty(mea.lib.mea_bwd_workspace_size(B, M, Hq, K), dtype=torch.uint8, device=DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for st in (mea.BWD_PREP, mea.BWD_MAIN, mea.BWD_DQ):
        mea.mea_bwd(q, k, v, out, dout, lse, bias=p.bias, scale=p.scale, alibi=True, dq=dq,
                    dk=dk, dv=dv, workspace=ws, stages=st)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    assert torch.equal(full[1], dk) and torch.equal(full[2], dv)
    a, b = full[0].float(), dq.float()
    assert ((a - b).abs() <= 2.0 ** -7 * a.abs() + 1e-6).all()
