"""Parity of the split-KV decode path (mea_decode, through the C ABI) with the
fp64 oracle's decode definition on the same seeded inputs."""
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


def _run(mea, d: synth.Decode, max_kv_len=None):
    """One mea_decode with out, lse and the workspace between guard bands."""
    st = d.kv_seqstart.to(DEV)
    mkl = d.max_kv_len if max_kv_len is None else max_kv_len
    go = Guarded((d.B, 1, d.Hq, d.K), d.q.dtype, DEV, fill=float("nan"))
    gl = Guarded((d.B, d.Hq), torch.float32, DEV, fill=float("nan"))
    gw = Guarded((max(1, mea.mea_decode_workspace_size(d.B, d.Hq, d.Hkv, d.K, mkl)),),
                 torch.uint8, DEV)
    out, lse = mea.mea_decode(d.q.to(DEV), d.k_cache.to(DEV), d.v_cache.to(DEV), st, mkl,
                              scale=d.scale, alibi=d.alibi, out=go.t, lse=gl.t, workspace=gw.t)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    go.check(d.name + " out")
    gl.check(d.name + " lse")
    gw.check(d.name + " workspace")
    return out, lse


def _check(mea, orc, d: synth.Decode):
    out, lse = _run(mea, d)
    ref_o, ref_l = orc.decode(d.q, d.k_cache, d.v_cache, d.kv_seqstart, scale=d.scale,
                              alibi=d.alibi)
    assert_out_close(out[:, 0], ref_o, d.name)
    assert_lse_close(lse, ref_l, d.name)


RAGGED = [0, 1, 63, 64, 65, 511, 512, 513, 1500, 2047]


@pytest.mark.parametrize("alibi", [False, True])
@pytest.mark.parametrize("K,dtype,Hq,Hkv", [(128, "bf16", 8, 2), (64, "f16", 4, 4),
                                            (128, "f16", 16, 2), (64, "bf16", 6, 2)])
def test_decode_ragged(mea, orc, alibi, K, dtype, Hq, Hkv):
    d = synth.make_decode(f"dec_{K}_{dtype}_{Hq}_{Hkv}_a{alibi}", RAGGED, Hq, Hkv, K, dtype,
                          seed=100 + K + Hq, alibi=alibi)
    _check(mea, orc, d)


def test_decode_larger_bound_than_needed(mea, orc):
    """max_kv_len may exceed every length (extra splits exit early)."""
    d = synth.make_decode("dec_bound", [5, 700, 1024], 8, 2, 128, "bf16", seed=7)
    out, lse = _run(mea, d, max_kv_len=5000)
    ref_o, ref_l = orc.decode(d.q, d.k_cache, d.v_cache, d.kv_seqstart, scale=d.scale)
    assert_out_close(out[:, 0], ref_o, "bound")
    assert_lse_close(lse, ref_l, "bound")


def test_decode_is_last_row_of_prefill(mea):
    """GPU decode equals the last row of the GPU causal prefill on the same keys."""
    lens = [300, 1000]
    d = synth.make_decode("dec_vs_prefill", lens, 8, 2, 128, "bf16", seed=9)
    out, _ = _run(mea, d)
    st = d.kv_seqstart
    for b, n in enumerate(lens):
        qp = torch.randn(1, n, 8, 128, dtype=torch.bfloat16)
        qp[0, n - 1] = d.q[b, 0]
        ks = d.k_cache[st[b]:st[b + 1]][None].to(DEV)
        vs = d.v_cache[st[b]:st[b + 1]][None].to(DEV)
        o, _ = mea.mea_fwd(qp.to(DEV), ks, vs, bias="causal", scale=d.scale)
        torch.cuda.synchronize()
        assert (o[0, n - 1].float() - out[b, 0].float()).abs().max().item() < 4e-3


def test_decode_full_workload(mea, orc):
    """B=64, lengths U[512, 8192], Hq=32, Hkv=8, K=128, bf16 -- every output."""
    d = synth.decode_step()
    _check(mea, orc, d)
