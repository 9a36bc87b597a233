"""Parity of block-sparse prefill (mea_fwd_block_sparse, through the C ABI) with
the fp64 oracle's block-sparse attention on the same seeded inputs and masks.
Same tolerances as the dense forward (parity_util)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import BIAS_CODE, Guarded, assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
BLK = 128


@pytest.fixture(scope="module")
def mea():
    import memory_efficient_exact_mea_b200 as m

    assert m.lib.mea_sparse_block_size() == BLK
    return m


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _run(mea, p, mask):
    """One mea_fwd_block_sparse with out and lse between guard bands."""
    go = Guarded((p.B, p.M, p.Hq, p.K), p.q.dtype, DEV, fill=float("nan"))
    gl = Guarded((p.B, p.Hq, p.M), torch.float32, DEV, fill=float("nan"))
    out, lse = mea.mea_fwd_block_sparse(p.q.to(DEV), p.k.to(DEV), p.v.to(DEV), mask.to(DEV),
                                        bias=p.bias, scale=p.scale, alibi=p.alibi, out=go.t,
                                        lse=gl.t)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    go.check(p.name + " out")
    gl.check(p.name + " lse")
    return out, lse


def _full_mask(mask, B, Hq):
    return mask.expand(B, Hq, *mask.shape[2:]).contiguous()


def _check(mea, orc, p, mask, what):
    out, lse = _run(mea, p, mask)
    ro, rl = orc.attention_block_sparse(p.q, p.k, p.v, _full_mask(mask, p.B, p.Hq), BLK, BLK,
                                        bias=BIAS_CODE[p.bias], scale=p.scale, alibi=p.alibi)
    assert_out_close(out, ro, what)
    assert_lse_close(lse, rl, what)
    return out, lse


# Both TMEM layouts: separate P (K=64 fp16) and P over S (bf16 or K=128).
@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16"), (64, "bf16")])
@pytest.mark.parametrize("bias", ["none", "causal"])
@pytest.mark.parametrize("density", [0.3, 0.7])
def test_random_masks(mea, orc, K, dtype, bias, density):
    """Ragged sizes (several query tiles per CTA, a partial last key block);
    masks drawn per (batch, head) so the two query tiles of a CTA differ."""
    p = synth.make_prefill(f"bs_{K}_{dtype}_{bias}", 2, 700, 650, 4, 2, K, dtype, bias,
                           alibi=(bias == "causal"), seed=300 + K)
    mask = synth.block_mask(2, 4, 700, 650, BLK, density, seed=301 + int(10 * density))
    _check(mea, orc, p, mask, f"{p.name} d={density}")


@pytest.mark.parametrize("M,N", [(300, 900), (900, 300), (1, 500), (129, 129)])
def test_rectangular_causal(mea, orc, M, N):
    p = synth.make_prefill(f"bs_rect_{M}x{N}", 1, M, N, 2, 2, 64, "f16", "causal", seed=310)
    mask = synth.block_mask(1, 2, M, N, BLK, 0.6, seed=311)
    _check(mea, orc, p, mask, p.name)


def test_all_ones_equals_dense(mea, orc):
    """An all-ones mask computes the tiles mea_fwd computes.  Without a causal
    mask both walk the key tiles in the same order: bit-identical results.  Under
    a causal mask the dense kernel walks down from the diagonal while the
    block-sparse one walks up, so the sums are reordered: both are checked
    against the oracle and against each other at the forward's tolerance."""
    for K, dtype, bias in ((64, "f16", "none"), (128, "bf16", "causal")):
        p = synth.make_prefill(f"bs_ones_{K}", 2, 520, 520, 4, 4, K, dtype, bias, seed=320)
        mask = torch.ones((1, 1, 5, 5), dtype=torch.uint8)
        out, lse = _check(mea, orc, p, mask, p.name)
        d_out, d_lse = mea.mea_fwd(p.q.to(DEV), p.k.to(DEV), p.v.to(DEV), bias=bias,
                                   scale=p.scale)
        if bias == "none":
            assert torch.equal(out, d_out) and torch.equal(lse, d_lse)
        else:
            assert_out_close(d_out.cpu().double(), out.cpu().double(), "dense vs all-ones")
            assert_lse_close(d_lse.cpu().double(), lse.cpu().double(), "dense vs all-ones")


def test_all_zero_and_empty_rows(mea, orc):
    """A zero mask leaves every row empty (out 0, lse -inf); a zero block row
    empties just those 128 rows."""
    p = synth.make_prefill("bs_zero", 1, 384, 384, 2, 2, 64, "f16", "none", seed=330)
    out, lse = _run(mea, p, torch.zeros((1, 2, 3, 3), dtype=torch.uint8))
    assert not out.any() and torch.isneginf(lse).all()
    mask = torch.ones((1, 2, 3, 3), dtype=torch.uint8)
    mask[0, 1, 1, :] = 0
    out, lse = _check(mea, orc, p, mask, "zero block row")
    assert torch.isneginf(lse[0, 1, 128:256]).all()


def test_broadcast_mask(mea, orc):
    """One [1, 1, ., .] mask shared by every batch and head (stride 0)."""
    p = synth.make_prefill("bs_bcast", 3, 400, 400, 4, 1, 128, "f16", "causal", seed=340)
    mask = synth.block_mask(1, 1, 400, 400, BLK, 0.5, seed=341, keep_diagonal=True)
    _check(mea, orc, p, mask, p.name)


def test_full_size_sampled(mea, orc):
    """The benchmarked block-sparse workload (M=N=4096), sampled rows."""
    p, mask = synth.block_sparse_noncausal()
    out, lse = _run(mea, p, mask)
    rng = np.random.default_rng(6)
    rows = np.array([(int(rng.integers(p.B)), int(rng.integers(p.M)), int(rng.integers(p.Hq)))
                     for _ in range(192)] + [(0, 0, 0), (7, 4095, 15), (3, 128, 5)], dtype=np.int64)
    ro, rl = orc.attention_block_sparse(p.q, p.k, p.v, mask, BLK, BLK, bias=BIAS_CODE[p.bias],
                                        scale=p.scale, rows=rows)
    b, i, h = rows[:, 0], rows[:, 1], rows[:, 2]
    assert_out_close(out.cpu()[b, i, h], ro, p.name)
    assert_lse_close(lse.cpu()[b, h, i], rl, p.name)
