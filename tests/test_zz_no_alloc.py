"""The allocation-free decode entry point, mea_decode_noalloc, called through the
C ABI.  It is for callers that cannot allocate device memory at the point of the
call (an embedded runtime that owns all device memory, or a serving loop that
must not call cudaMalloc after start-up).  Its results must equal those of
mea_decode, which takes a caller-provided workspace, within the tolerances the
other parity tests use; it is called twice in a row on different problems, so
the second call also shows that the shared scratch array's stale contents from
the first call do not leak into the result."""
import ctypes

import pytest
import torch

import synth
from parity_util import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

DEV = "cuda"
MEA_ERR_WORKSPACE = -3


def _entry_point():
    import memory_efficient_exact_mea_b200 as mea

    lib = ctypes.CDLL(mea.LIB_PATH)
    fn = lib.mea_decode_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.restype = i
    fn.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, ctypes.c_float, vp]
    return mea, fn


def _call(fn, d, q, kc, vc, st, out, lse):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
              ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(st.data_ptr()),
              ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
              d.B, d.Hq, d.Hkv, d.K, kc.shape[0], d.max_kv_len,
              1 if d.dtype == "bf16" else 0, int(d.alibi), d.scale, stream)


def test_noalloc_matches_workspace_entry_point():
    mea, fn = _entry_point()
    problems = [
        synth.make_decode("noalloc_a", [0, 1, 65, 513, 1500, 4100], 8, 2, 128, "bf16", seed=301),
        synth.make_decode("noalloc_b", [700, 33, 2048], 16, 4, 64, "f16", seed=302, alibi=True),
    ]
    for d in problems:  # two calls in a row, different shapes
        q, kc, vc = d.q.to(DEV), d.k_cache.to(DEV), d.v_cache.to(DEV)
        st = d.kv_seqstart.to(DEV)
        ref_out, ref_lse = mea.mea_decode(q, kc, vc, st, d.max_kv_len, scale=d.scale,
                                          alibi=d.alibi)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((d.B, d.Hq), float("nan"), dtype=torch.float32, device=DEV)
        assert _call(fn, d, q, kc, vc, st, out, lse) == 0
        torch.cuda.synchronize()
        assert mea.read_device_status() == 0
        assert_out_close(out, ref_out, d.name)
        assert_lse_close(lse, ref_lse, d.name)


def test_noalloc_rejects_problems_beyond_its_scratch():
    """B=64, Hq=64, K=128, max_kv_len=65536 needs 270 MB of partials (> 32 MiB):
    rejected on the host with MEA_ERR_WORKSPACE, nothing launched."""
    mea, fn = _entry_point()
    d = synth.Decode("too_big", 64, 64, 8, 128, "bf16", 0, [65536] * 64)
    assert mea.mea_decode_workspace_size(64, 64, 8, 128, 65536) > 32 << 20
    q = torch.zeros(64, 1, 64, 128, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(8, 8, 128, dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(65, dtype=torch.int32, device=DEV)
    out = torch.zeros_like(q)
    lse = torch.zeros(64, 64, dtype=torch.float32, device=DEV)
    assert _call(fn, d, q, kc, kc, st, out, lse) == MEA_ERR_WORKSPACE
