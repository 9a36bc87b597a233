"""The allocation-free decode entry point, mea_decode_noalloc, called through the
C ABI.  It is for callers that cannot allocate device memory at the point of the
call (an embedded runtime that owns all device memory, or a serving loop that
must not call cudaMalloc after start-up).  Its results must equal those of
mea_decode, which takes a caller-provided workspace, and those of the fp64
oracle, within the tolerances the other parity tests use.  It is called several
times in a row on problems of different sizes, and once with offsets the device
rejects, so the later calls also show that the shared scratch array's stale
contents from earlier calls never leak into a result."""
import ctypes

import pytest
import torch

import oracle
import synth
from parity_util import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

DEV = "cuda"
MEA_ERR_WORKSPACE = -3
MEA_ERR_INVALID_ARG = -1


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


def _run_and_compare(mea, fn, orc, d):
    """One no-alloc call, checked against mea_decode and against the oracle."""
    q, kc, vc = d.q.to(DEV), d.k_cache.to(DEV), d.v_cache.to(DEV)
    st = d.kv_seqstart.to(DEV)
    ref_out, ref_lse = mea.mea_decode(q, kc, vc, st, d.max_kv_len, scale=d.scale, alibi=d.alibi)
    out = torch.full_like(q, float("nan"))
    lse = torch.full((d.B, d.Hq), float("nan"), dtype=torch.float32, device=DEV)
    assert _call(fn, d, q, kc, vc, st, out, lse) == 0
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    assert_out_close(out, ref_out, d.name)
    assert_lse_close(lse, ref_lse, d.name)
    o_ref, l_ref = orc.decode(d.q, d.k_cache, d.v_cache, d.kv_seqstart, scale=d.scale,
                              alibi=d.alibi)
    assert_out_close(out[:, 0], o_ref, d.name + " vs oracle")
    assert_lse_close(lse, l_ref, d.name + " vs oracle")


def test_noalloc_matches_workspace_entry_point():
    """Calls in a row on problems of different sizes: a moderate one, a smaller
    one (reads less of the array than the first wrote), then a larger one with a
    longer max_kv_len (reads further than either earlier call wrote)."""
    mea, fn = _entry_point()
    orc = oracle.get()
    problems = [
        synth.make_decode("noalloc_a", [0, 1, 65, 513, 1500, 4100], 8, 2, 128, "bf16", seed=301),
        synth.make_decode("noalloc_b", [700, 33, 2048], 16, 4, 64, "f16", seed=302, alibi=True),
        synth.make_decode("noalloc_c", [9000, 3, 512, 1025, 6000, 7, 4000, 8191], 32, 8, 128,
                          "bf16", seed=303),
    ]
    for d in problems:
        _run_and_compare(mea, fn, orc, d)


def test_noalloc_after_rejected_offsets():
    """A call whose kv_seqstart runs past the cache: the device-side checks skip
    that sequence (out 0, lse NaN, MEA_ERR_INVALID_ARG in the status word), the
    valid sequences are still right, and the next call is unaffected."""
    mea, fn = _entry_point()
    orc = oracle.get()
    d = synth.make_decode("noalloc_bad", [300, 1100, 50], 8, 2, 128, "bf16", seed=304)
    q, kc, vc = d.q.to(DEV), d.k_cache.to(DEV), d.v_cache.to(DEV)
    st_host = d.kv_seqstart.clone()
    st_host[-1] += 40  # the last sequence claims 40 rows past the end of the cache
    st = st_host.to(DEV)
    out = torch.full_like(q, float("nan"))
    lse = torch.zeros((d.B, d.Hq), dtype=torch.float32, device=DEV)
    d_bad = synth.Decode(d.name, d.B, d.Hq, d.Hkv, d.K, d.dtype, d.seed, [300, 1100, 90])
    assert _call(fn, d_bad, q, kc, vc, st, out, lse) == 0
    torch.cuda.synchronize()
    assert mea.read_device_status() == MEA_ERR_INVALID_ARG
    assert mea.read_device_status() == 0
    assert torch.all(out[2] == 0) and torch.all(torch.isnan(lse[2]))
    o_ref, l_ref = orc.decode(d.q, d.k_cache, d.v_cache, d.kv_seqstart, scale=d.scale)
    assert_out_close(out[:2, 0], o_ref[:2], "valid rows of the rejected call")
    assert_lse_close(lse[:2], l_ref[:2], "valid rows of the rejected call")
    _run_and_compare(mea, fn, orc, synth.make_decode("noalloc_after", [2000, 5, 777], 8, 2, 128,
                                                     "bf16", seed=305))


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
