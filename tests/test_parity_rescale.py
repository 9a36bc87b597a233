"""Parity of every forward instance family with the fp64 oracle on inputs whose
row maxima move across key tiles, so that the running-max update and the
rescale of the output accumulator actually run ("FlashAttention (2022)", "Il
trucco della softmax che non ha bisogno di vedere tutto": each new block of
keys updates the running maximum and rescales what was accumulated so far).

The kernels keep a stale reference maximum until a tile's maximum exceeds it by
more than 2^8 (in log2 units), so plain N(0,1) inputs at scale 1/sqrt(K) never
leave the first tile's reference.  The inputs here do:
  rising   keys multiplied by 1 .. 16 along each sequence's key positions: the
           maximum climbs by more than 2^8 many times along a row;
  falling  keys multiplied by 16 .. 1: the maximum sits in the first tiles and
           the later weights underflow;
  large    q and k times 4 at scale 1: |scores| of a few hundred to about a
           thousand, exercising fp32 logits far from zero;
  steps    scores constant per 128-key tile, moving by exactly 8, 7.9375,
           8.0625, ... log2 units from tile to tile (scale = ln 2, so a score is
           its log2 logit), around the threshold where the reference moves.
Dense causal instances walk a unit's key tiles from the diagonal down, so for
them "falling" is the shape whose maximum climbs; the step shapes run with both
signs.
Every instance family without ALiBi is covered (ALiBi's growing bias already
moves the maximum): the persistent K=64 fp16 non-causal instance with more
units than SMs, K=64 fp16 causal (P in its own tensor-memory columns), K=128
bf16 / K=64 bf16 / K=128 fp16 (P written over S, bf16 as hi + lo), block-sparse,
chunked prefill and packed variable-length batches.  Every element of out and
lse is compared (parity_util tolerances), and every output sits between guard
bands that must come back untouched."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import BIAS_CODE, Guarded, assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
LN2_F32 = float(np.float32(np.log(2.0)))  # scale whose fp32 product with log2(e) is 1
STEPS = [8.0, 7.9375, 8.0625, 8.0, -30.0, 8.0, 16.0, 7.9375, 0.5]


@pytest.fixture(scope="module")
def mea():
    import memory_efficient_exact_mea_b200 as m

    return m


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _shape(p: synth.Prefill, how: str):
    """Apply one of the score shapes; returns (problem, scale)."""
    if how == "rising":
        return synth.ramp_keys(p, 1.0, 16.0), p.scale
    if how == "falling":
        return synth.ramp_keys(p, 16.0, 1.0), p.scale
    if how == "large":
        return synth.amplify(p, 4.0), 1.0
    raise ValueError(how)


def _fwd(mea, p, scale, block_mask=None):
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    go = Guarded((p.B, p.M, p.Hq, p.K), q.dtype, DEV, fill=float("nan"))
    gl = Guarded((p.B, p.Hq, p.M), torch.float32, DEV, fill=float("nan"))
    if block_mask is not None:
        mea.mea_fwd_block_sparse(q, k, v, block_mask.to(DEV), bias=p.bias, scale=scale,
                                 out=go.t, lse=gl.t)
    else:
        kw = {}
        if p.bias.startswith("blockdiag"):
            kw = dict(seqstart_q=p.seqstart_q.to(DEV), seqstart_k=p.seqstart_k.to(DEV))
        mea.mea_fwd(q, k, v, bias=p.bias, scale=scale, alibi=p.alibi, out=go.t, lse=gl.t, **kw)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    go.check(p.name + " out")
    gl.check(p.name + " lse")
    return go.t, gl.t


def _check_dense(mea, orc, p, scale):
    out, lse = _fwd(mea, p, scale)
    ro, rl = orc.attention(p.q, p.k, p.v, bias=BIAS_CODE[p.bias], scale=scale, alibi=p.alibi,
                           seqstart_q=p.seqstart_q, seqstart_k=p.seqstart_k)
    assert_out_close(out, ro, p.name)
    assert_lse_close(lse, rl, p.name)


# (name, B, M, N, Hq, Hkv, K, dtype, bias): one per instance family of mea_fwd.
DENSE = [
    # persistent instance: 4 query blocks x 20 heads x 2 batches = 160 units > 148 SMs
    ("persist_k64_f16_none", 2, 1024, 1000, 20, 20, 64, "f16", "none"),
    ("sepP_k64_f16_causal", 2, 1000, 1000, 4, 2, 64, "f16", "causal"),
    ("alias_k128_bf16_none", 2, 1000, 900, 4, 2, 128, "bf16", "none"),
    ("alias_k128_bf16_causal", 2, 1000, 1000, 4, 2, 128, "bf16", "causal"),
    ("alias_k64_bf16_none", 2, 700, 1000, 4, 4, 64, "bf16", "none"),
    ("alias_k128_f16_causal", 2, 900, 1000, 4, 1, 128, "f16", "causal"),
]


@pytest.mark.parametrize("how", ["rising", "falling", "large"])
@pytest.mark.parametrize("case", DENSE, ids=[c[0] for c in DENSE])
def test_dense_moving_max(mea, orc, case, how):
    name, B, M, N, Hq, Hkv, K, dtype, bias = case
    p = synth.make_prefill(name, B, M, N, Hq, Hkv, K, dtype, bias, seed=500 + M + K)
    p, scale = _shape(p, how)
    _check_dense(mea, orc, p, scale)


STEP_CASES = [(64, "f16", "none"), (64, "f16", "causal"), (128, "bf16", "none"),
              (128, "bf16", "causal"), (64, "bf16", "none"), (128, "f16", "causal")]


@pytest.mark.parametrize("sign", [1.0, -1.0])
@pytest.mark.parametrize("noise", [0.0, 0.05])
@pytest.mark.parametrize("K,dtype,bias", STEP_CASES)
def test_threshold_steps(mea, orc, K, dtype, bias, noise, sign):
    """Tile-to-tile jumps of exactly 8 (kept stale: P reaches 2^8), 7.9375 (kept),
    8.0625 (moved), a fall of 30 and a rise of 16, in rotated orders per batch;
    with noise the rows straddle the threshold differently.  The negated steps
    give the same jumps to a kernel that walks the key tiles downwards (dense
    causal instances)."""
    steps = [sign * s for s in STEPS]
    p = synth.tile_step_scores(f"steps_{K}_{dtype}_{bias}_n{noise}_s{sign:+.0f}", 3, 1100, 2, K,
                               dtype, steps, 128, seed=520 + K, bias=bias, noise=noise)
    _check_dense(mea, orc, p, LN2_F32)


@pytest.mark.parametrize("how", ["rising", "falling", "large"])
@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16")])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_moving_max(mea, orc, K, dtype, causal, how):
    lens = [1, 127, 129, 300, 700, 0, 1030]
    p = synth.make_varlen(f"varlen_{K}_{dtype}_c{causal}", lens, 4, 2, K, dtype, causal,
                          seed=540 + K)
    p, scale = _shape(p, how)
    _check_dense(mea, orc, p, scale)


@pytest.mark.parametrize("how", ["rising", "large"])
@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16"), (64, "bf16")])
@pytest.mark.parametrize("bias", ["none", "causal"])
def test_block_sparse_moving_max(mea, orc, K, dtype, bias, how):
    p = synth.make_prefill(f"bs_{K}_{dtype}_{bias}", 2, 700, 1000, 4, 2, K, dtype, bias,
                           seed=560 + K)
    p, scale = _shape(p, how)
    mask = synth.block_mask(2, 4, 700, 1000, 128, 0.6, seed=561, keep_diagonal=True)
    out, lse = _fwd(mea, p, scale, block_mask=mask)
    ro, rl = orc.attention_block_sparse(p.q, p.k, p.v, mask, 128, 128, bias=BIAS_CODE[bias],
                                        scale=scale)
    assert_out_close(out, ro, p.name)
    assert_lse_close(lse, rl, p.name)


@pytest.mark.parametrize("how", ["rising", "falling", "large"])
@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16"), (64, "bf16"), (128, "f16")])
@pytest.mark.parametrize("causal", [True, False])
def test_chunk_moving_max(mea, orc, K, dtype, causal, how):
    c = synth.make_chunk(f"chunk_{K}_{dtype}_c{causal}", [0, 1, 128, 200, 1000], 300, 1400, 4, 2,
                         K, dtype, causal, seed=580 + K)
    scale = c.scale
    if how == "rising":
        c = synth.ramp_chunk_keys(c, 1.0, 16.0)
    elif how == "falling":
        c = synth.ramp_chunk_keys(c, 16.0, 1.0)
    else:
        for t in ("q", "k_new", "k_cache"):
            setattr(c, t, (getattr(c, t).to(torch.float32) * 4.0).to(getattr(c, t).dtype))
        scale = 1.0
    kc, vc = c.k_cache.to(DEV), c.v_cache.to(DEV)
    cl = torch.tensor(c.past, dtype=torch.int32, device=DEV)
    go = Guarded((c.B, c.M, c.Hq, c.K), c.q.dtype, DEV, fill=0.0)
    gl = Guarded((c.B, c.Hq, c.M), torch.float32, DEV, fill=0.0)
    mea.mea_prefill_chunk(c.q.to(DEV), c.k_new.to(DEV), c.v_new.to(DEV), kc, vc, cl,
                          causal=causal, scale=scale, out=go.t, lse=gl.t)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    go.check(c.name + " out")
    gl.check(c.name + " lse")
    ro, rl, rkc, rvc = orc.prefill_chunk(c.q, c.k_new, c.v_new, c.k_cache, c.v_cache, c.past,
                                         causal=causal, scale=scale)
    assert_out_close(go.t, ro, c.name)
    assert_lse_close(gl.t, rl, c.name)
    assert np.array_equal(kc.cpu().to(torch.float64).numpy(), rkc), f"{c.name}: k cache"
    assert np.array_equal(vc.cpu().to(torch.float64).numpy(), rvc), f"{c.name}: v cache"


@pytest.mark.parametrize("K,dtype,bias", [(64, "f16", "none"), (128, "bf16", "causal")])
def test_backward_after_moving_max(mea, K, dtype, bias):
    """The backward recomputes the weights from the forward's lse; with rising
    keys that lse comes out of many reference moves."""
    p = synth.ramp_keys(synth.make_prefill(f"bwd_rise_{K}_{dtype}_{bias}", 2, 300, 300, 4, 2, K,
                                           dtype, bias, seed=600 + K), 1.0, 16.0)
    dout = synth.randn(tuple(p.q.shape), p.dtype, synth.generator(p.seed + 17))
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    out, lse = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale)
    gq, gk, gv = (Guarded(tuple(t.shape), t.dtype, DEV) for t in (q, k, v))
    mea.mea_bwd(q, k, v, out, dout.to(DEV), lse, bias=p.bias, scale=p.scale, dq=gq.t, dk=gk.t,
                dv=gv.t)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    for g, nm in ((gq, "dq"), (gk, "dk"), (gv, "dv")):
        g.check(f"{p.name} {nm}")
    refs = oracle.get().attention_bwd(p.q, p.k, p.v, dout, bias=BIAS_CODE[p.bias], scale=p.scale)
    from test_parity_bwd import _assert_grad

    for g, r, nm in zip((gq.t, gk.t, gv.t), refs, ("dq", "dk", "dv")):
        _assert_grad(g, r, p.dtype, f"{p.name} {nm}")
