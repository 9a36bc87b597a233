"""Failure detection on the GPU without a fault: a device wait that can never be
satisfied runs out its (short) limit, the kernel records MEA_ERR_DEVICE_TIMEOUT
in the status word and returns, and the context keeps working."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import assert_lse_close, assert_out_close

MEA_ERR_DEVICE_TIMEOUT = -5


def _selftest():
    import memory_efficient_exact_mea_b200 as mea

    fn = mea.lib.mea_selftest_timeout
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int, ctypes.c_void_p]
    return mea, fn


def test_selftest_rejects_bad_limits():
    """Host-side argument checks; nothing is launched."""
    _, fn = _selftest()
    assert fn(0, None) == -1
    assert fn(-5, None) == -1
    assert fn(20_000_000, None) == -1


@pytest.mark.gpu
def test_timed_out_wait_is_reported_and_context_survives():
    mea, fn = _selftest()
    assert mea.read_device_status(clear=True) == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert fn(50_000, stream) == 0  # 50 ms limit
    assert mea.read_device_status(clear=True) == MEA_ERR_DEVICE_TIMEOUT
    assert mea.read_device_status(clear=False) == 0
    # The context still runs the real kernels correctly.
    p = synth.make_prefill("after_timeout", 1, 200, 200, 2, 2, 64, "f16", "causal", seed=90)
    out, lse = mea.mea_fwd(p.q.cuda(), p.k.cuda(), p.v.cuda(), bias="causal", scale=p.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.get().attention(p.q, p.k, p.v, bias=oracle.BIAS_CAUSAL, scale=p.scale)
    assert_out_close(out, ref_o, "after timeout")
    assert_lse_close(lse, ref_l, "after timeout")
    assert mea.read_device_status() == 0
    assert np.isfinite(lse.cpu().numpy()).all()
