"""Parity of chunked prefill with the fused cache append (mea_prefill_chunk,
through the C ABI) with the fp64 oracle's prefill_chunk on the same seeded
inputs: out and lse within the forward's tolerances, the cache after the call
bit-exact (the append is a copy)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import Guarded, assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def mea():
    import memory_efficient_exact_mea_b200 as m

    return m


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _run(mea, c: synth.Chunk, kc=None, vc=None):
    kc = c.k_cache.to(DEV) if kc is None else kc
    vc = c.v_cache.to(DEV) if vc is None else vc
    cl = torch.tensor(c.past, dtype=torch.int32, device=DEV)
    ql = torch.tensor(c.q_lens, dtype=torch.int32, device=DEV)
    go = Guarded((c.B, c.M, c.Hq, c.K), c.q.dtype, DEV, fill=0.0)
    gl = Guarded((c.B, c.Hq, c.M), torch.float32, DEV, fill=123.0)
    out, lse = go.t, gl.t
    mea.mea_prefill_chunk(c.q.to(DEV), c.k_new.to(DEV), c.v_new.to(DEV), kc, vc, cl, ql,
                          causal=c.causal, scale=c.scale, alibi=c.alibi, out=out, lse=lse)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    go.check(c.name + " out")
    gl.check(c.name + " lse")
    return out, lse, kc, vc


def _check(mea, orc, c: synth.Chunk, what):
    out, lse, kc, vc = _run(mea, c)
    ro, rl, rkc, rvc = orc.prefill_chunk(c.q, c.k_new, c.v_new, c.k_cache, c.v_cache, c.past,
                                         q_len=c.q_lens, causal=c.causal, scale=c.scale,
                                         alibi=c.alibi)
    for b, n in enumerate(c.q_lens):
        assert_out_close(out[b, :n], ro[b, :n], f"{what} b={b}")
        assert_lse_close(lse[b, :, :n], rl[b, :, :n], f"{what} b={b}")
        assert not out[b, n:].any() and (lse[b, :, n:] == 123.0).all(), "padding rows written"
    assert np.array_equal(kc.cpu().to(torch.float64).numpy(), rkc), f"{what}: k cache"
    assert np.array_equal(vc.cpu().to(torch.float64).numpy(), rvc), f"{what}: v cache"


@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16"), (64, "bf16"), (128, "f16")])
@pytest.mark.parametrize("causal", [True, False])
def test_chunk(mea, orc, K, dtype, causal):
    """Past lengths on and off tile boundaries (0, 1, 128, 200, 1000); a chunk of
    300 rows (several query tiles, a ragged last key tile)."""
    c = synth.make_chunk(f"chunk_{K}_{dtype}_c{causal}", [0, 1, 128, 200, 1000], 300, 1400, 4,
                         2, K, dtype, causal, seed=400 + K, alibi=causal)
    _check(mea, orc, c, c.name)


def test_ragged_chunks(mea, orc):
    """Per-sequence chunk lengths (0, 1, 127, 129, M) with GQA and ALiBi."""
    c = synth.make_chunk("chunk_ragged", [5, 300, 0, 77, 128], 260, 600, 8, 2, 128, "bf16",
                         True, seed=410, q_lens=[0, 1, 127, 129, 260], alibi=True)
    _check(mea, orc, c, c.name)


def test_stale_cache_rows_are_never_read(mea, orc):
    """Cache rows at and after past hold NaN before the call: the results and
    the appended rows must not see them."""
    c = synth.make_chunk("chunk_nan", [130, 7], 200, 512, 4, 4, 64, "f16", True, seed=420)
    for b, p in enumerate(c.past):
        c.k_cache[b, p:] = float("nan")
        c.v_cache[b, p:] = float("nan")
    out, lse, kc, vc = _run(mea, c)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    ro, rl, rkc, _ = orc.prefill_chunk(c.q, c.k_new, c.v_new, c.k_cache, c.v_cache, c.past,
                                       causal=True, scale=c.scale)
    assert_out_close(out, ro, "nan-filled cache")
    assert_lse_close(lse, rl, "nan-filled cache")
    got = kc.cpu().to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(rkc)) and np.array_equal(
        np.nan_to_num(got), np.nan_to_num(rkc))


def test_two_chunks_equal_one_prefill(mea):
    """Two chunks in a row through the same cache give (within rounding) the
    rows of one causal mea_fwd over the whole sequence."""
    c = synth.make_chunk("chunk_pair", [0, 0], 384, 800, 4, 2, 128, "bf16", True, seed=430)
    q, kn, vn = c.q.to(DEV), c.k_new.to(DEV), c.v_new.to(DEV)
    kc, vc = c.k_cache.to(DEV), c.v_cache.to(DEV)
    zero = torch.zeros(2, dtype=torch.int32, device=DEV)
    split = torch.tensor([100, 250], dtype=torch.int32, device=DEV)
    o1, l1 = mea.mea_prefill_chunk(q, kn, vn, kc, vc, zero, split, scale=c.scale)
    # second chunk: rows split[b].. of the sequence, shifted to the start
    q2, k2, v2 = (torch.zeros_like(x) for x in (q, kn, vn))
    for b, a in enumerate((100, 250)):
        q2[b, :384 - a], k2[b, :384 - a], v2[b, :384 - a] = q[b, a:], kn[b, a:], vn[b, a:]
    rest = torch.tensor([284, 134], dtype=torch.int32, device=DEV)
    o2, l2 = mea.mea_prefill_chunk(q2, k2, v2, kc, vc, split, rest, scale=c.scale)
    of, lf = mea.mea_fwd(q, kn, vn, bias="causal", scale=c.scale)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    for b, a in enumerate((100, 250)):
        assert_out_close(o1[b, :a], of[b, :a].double(), "first chunk")
        assert_out_close(o2[b, :384 - a], of[b, a:].double(), "second chunk")
        assert_lse_close(l2[b, :, :384 - a], lf[b, :, a:].double(), "second chunk lse")
        assert torch.equal(kc[b, :384], kn[b]) and torch.equal(vc[b, :384], vn[b])


def test_overflowing_chunk_is_reported(mea):
    """past + n beyond the cache: that sequence is skipped and the device status
    word reports an invalid argument (no fault); the others are computed."""
    c = synth.make_chunk("chunk_over", [10, 250], 64, 256, 2, 2, 64, "f16", True, seed=440)
    kc, vc = c.k_cache.to(DEV), c.v_cache.to(DEV)
    cl = torch.tensor(c.past, dtype=torch.int32, device=DEV)
    out, _ = mea.mea_prefill_chunk(c.q.to(DEV), c.k_new.to(DEV), c.v_new.to(DEV), kc, vc, cl,
                                   scale=c.scale)
    assert mea.read_device_status() == -1
    assert torch.isfinite(out[0]).all()
    assert torch.equal(kc[1].cpu(), c.k_cache[1])


def test_full_size_sampled(mea, orc):
    """The benchmarked chunk workload (B=8, 512-row chunks, 1k-8k cached rows);
    two of its sequences checked against the oracle."""
    c = synth.chunk_prefill()
    out, lse, kc, vc = _run(mea, c)
    for b in (0, 5):
        sub = synth.Chunk(c.name, 1, c.M, c.cap, c.Hq, c.Hkv, c.K, c.dtype, c.causal,
                          [c.past[b]], [c.M], c.alibi, c.seed, c.q[b:b + 1], c.k_new[b:b + 1],
                          c.v_new[b:b + 1], c.k_cache[b:b + 1], c.v_cache[b:b + 1])
        ro, rl, rkc, _ = orc.prefill_chunk(sub.q, sub.k_new, sub.v_new, sub.k_cache, sub.v_cache,
                                           sub.past, causal=True, scale=c.scale)
        assert_out_close(out[b], ro[0], f"{c.name} b={b}")
        assert_lse_close(lse[b], rl[0], f"{c.name} b={b}")
        p = c.past[b]
        assert np.array_equal(kc[b, p:p + c.M].cpu().to(torch.float64).numpy(), rkc[0, p:p + c.M])


@pytest.mark.parametrize("causal,alibi", [(False, False), (True, False), (True, True)])
def test_chunk_repeatable(mea, causal, alibi):
    """Ten launches on the same input give bit-identical outputs (a race between
    a TMEM load and its use would show as run-to-run differences)."""
    c = synth.make_chunk("chunk_rep", [0, 1, 128, 200, 1000], 300, 1400, 4, 2, 64, "f16", causal,
                         seed=450, alibi=alibi)
    first = None
    for _ in range(10):
        out, lse, _, _ = _run(mea, c)
        if first is None:
            first = (out, lse)
        else:
            assert torch.equal(out, first[0]) and torch.equal(lse, first[1])
