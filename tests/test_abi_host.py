"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/mea.h declares, and rejects bad arguments before any
launch with the documented status codes."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mea.h")


@pytest.fixture(scope="module")
def lib():
    import memory_efficient_exact_mea_b200 as m

    return m.lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mea_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("mea_fwd", "mea_decode", "mea_decode_workspace_size", "mea_status_string",
              "mea_read_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in mea.h but not exported"


def test_status_strings(lib):
    import memory_efficient_exact_mea_b200 as m

    assert m.status_string(0) == "ok"
    for code in (-1, -2, -3, -4, -5):
        assert m.status_string(code) not in ("", "unknown status")
    assert m.status_string(123) == "unknown status"
    assert lib.mea_version() >= 10000


def test_decode_workspace_size(lib):
    import memory_efficient_exact_mea_b200 as m

    C = m.mea_decode_chunk()
    assert C > 0
    # rows = B * Hq * splits; partial outputs K floats per row, lse one float per row,
    # each region rounded up to 256 bytes.
    for (B, Hq, K, L) in ((64, 32, 128, 8192), (3, 5, 64, 1), (1, 1, 128, C), (2, 4, 64, C + 1)):
        splits = -(-L // C)
        rows = B * Hq * splits
        r256 = lambda x: -(-x // 256) * 256  # noqa: E731
        assert m.mea_decode_workspace_size(B, Hq, 1, K, L) == r256(rows * K * 4) + r256(rows * 4)
    assert m.mea_decode_workspace_size(4, 8, 2, 128, 0) == 0
    assert m.mea_decode_workspace_size(-1, 8, 2, 128, 10) == 0


I64x3 = ctypes.c_int64 * 3


def _fwd(lib, **kw):
    a = dict(q=16, k=16, v=16, out=16, lse=None, B=1, M=8, N=8, Hq=2, Hkv=1, K=64,
             qs=I64x3(1024, 128, 64), ks=I64x3(512, 64, 64), vs=I64x3(512, 64, 64),
             os_=I64x3(1024, 128, 64), dtype=0, bias=0, sq=None, sk=None, ns=0, mq=0, mk=0,
             alibi=0, scale=0.125, stream=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return lib.mea_fwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["out"]), vp(a["lse"]),
                       a["B"], a["M"], a["N"], a["Hq"], a["Hkv"], a["K"], a["qs"], a["ks"],
                       a["vs"], a["os_"], a["dtype"], a["bias"], vp(a["sq"]), vp(a["sk"]),
                       a["ns"], a["mq"], a["mk"], a["alibi"], ctypes.c_float(a["scale"]),
                       vp(a["stream"]))


def test_fwd_rejects_bad_arguments(lib):
    INVALID, UNSUPPORTED = -1, -2
    assert _fwd(lib, Hq=3, Hkv=2) == INVALID          # Hq % Hkv
    assert _fwd(lib, Hkv=0) == INVALID
    assert _fwd(lib, M=-1) == INVALID
    assert _fwd(lib, dtype=7) == INVALID
    assert _fwd(lib, bias=9) == INVALID
    assert _fwd(lib, q=None) == INVALID
    assert _fwd(lib, k=None) == INVALID
    assert _fwd(lib, scale=float("nan")) == INVALID
    assert _fwd(lib, bias=2, B=2) == INVALID            # block-diagonal needs B == 1
    assert _fwd(lib, bias=3, sq=None, ns=1) == INVALID  # ... and offsets
    assert _fwd(lib, bias=2, sq=64, ns=1, N=9) == INVALID  # seqstart_k NULL needs M == N
    assert _fwd(lib, K=96) == UNSUPPORTED
    assert _fwd(lib, scale=-0.5) == UNSUPPORTED
    assert _fwd(lib, q=24) == UNSUPPORTED               # 16-byte alignment
    assert _fwd(lib, qs=I64x3(1024, 100, 64)) == UNSUPPORTED  # stride not a multiple of 8
    assert _fwd(lib, qs=I64x3(1024, 128, 0)) == UNSUPPORTED
    assert _fwd(lib, M=0) == 0                          # nothing to do
    assert _fwd(lib, B=0) == 0


def _dec(lib, **kw):
    a = dict(q=16, k=16, v=16, st=16, out=16, lse=None, B=2, Hq=8, Hkv=2, K=128, rows=100,
             maxlen=100, dtype=1, alibi=0, scale=0.1, ws=256, wsb=1 << 20, stream=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return lib.mea_decode(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["st"]), vp(a["out"]),
                          vp(a["lse"]), a["B"], a["Hq"], a["Hkv"], a["K"], a["rows"],
                          a["maxlen"], a["dtype"], a["alibi"], ctypes.c_float(a["scale"]),
                          vp(a["ws"]), a["wsb"], vp(a["stream"]))


def test_decode_rejects_bad_arguments(lib):
    INVALID, UNSUPPORTED, WORKSPACE = -1, -2, -3
    assert _dec(lib, Hq=6, Hkv=4) == INVALID
    assert _dec(lib, st=None) == INVALID
    assert _dec(lib, q=None) == INVALID
    assert _dec(lib, k=None) == INVALID
    assert _dec(lib, maxlen=-1) == INVALID
    assert _dec(lib, dtype=3) == INVALID
    assert _dec(lib, K=80) == UNSUPPORTED
    assert _dec(lib, Hq=32, Hkv=2) == UNSUPPORTED   # more than 8 query heads per kv head
    assert _dec(lib, out=8) == UNSUPPORTED
    assert _dec(lib, ws=None) == WORKSPACE
    assert _dec(lib, wsb=16) == WORKSPACE
    assert _dec(lib, ws=272) == WORKSPACE            # 256-byte alignment
    assert _dec(lib, B=0) == 0


def test_no_device_is_reported_not_crashed(lib):
    """Valid arguments on a host without a usable GPU come back as MEA_ERR_CUDA."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd(lib) == -4


def _bwd(lib, **kw):
    a = dict(q=16, k=16, v=16, out=16, do=16, lse=16, dq=16, dk=16, dv=16, B=2, M=100, N=100,
             Hq=8, Hkv=2, K=128, dtype=1, bias=1, sq=None, sk=None, ns=0, msq=0, msk=0, alibi=0,
             scale=0.1, ws=256, wsb=1 << 30, stream=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return lib.mea_bwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["out"]), vp(a["do"]),
                       vp(a["lse"]), vp(a["dq"]), vp(a["dk"]), vp(a["dv"]), a["B"], a["M"],
                       a["N"], a["Hq"], a["Hkv"], a["K"], a["dtype"], a["bias"], vp(a["sq"]),
                       vp(a["sk"]), a["ns"], a["msq"], a["msk"], a["alibi"],
                       ctypes.c_float(a["scale"]), vp(a["ws"]), a["wsb"], vp(a["stream"]))


def test_bwd_stages_rejects_bad_masks(lib):
    """mea_bwd_stages takes a nonzero OR of its three stage bits."""
    INVALID = -1
    vp = ctypes.c_void_p
    for stages in (0, 8, -1):
        rc = lib.mea_bwd_stages(vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16),
                                vp(16), 2, 100, 100, 8, 2, 128, 1, 1, None, None, 0, 0, 0, 0,
                                ctypes.c_float(0.1), vp(256), 1 << 30, stages, None)
        assert rc == INVALID, stages


def test_bwd_workspace_size():
    import memory_efficient_exact_mea_b200 as m

    r256 = lambda x: -(-x // 256) * 256  # noqa: E731
    for (B, M, Hq, K) in ((2, 100, 8, 128), (1, 1, 1, 64), (4, 4096, 32, 128)):
        rows = B * M * Hq
        assert m.lib.mea_bwd_workspace_size(B, M, Hq, K) == r256(rows * K * 4) + r256(rows * 4)
    assert m.lib.mea_bwd_workspace_size(-1, 4, 4, 64) == 0


def test_bwd_rejects_bad_arguments(lib):
    INVALID, UNSUPPORTED, WORKSPACE = -1, -2, -3
    assert _bwd(lib, Hq=3, Hkv=2) == INVALID
    assert _bwd(lib, N=-1) == INVALID
    assert _bwd(lib, dtype=5) == INVALID
    assert _bwd(lib, bias=4) == INVALID
    assert _bwd(lib, scale=float("nan")) == INVALID
    assert _bwd(lib, lse=None) == INVALID
    assert _bwd(lib, dk=None) == INVALID
    assert _bwd(lib, bias=2) == INVALID                   # block-diagonal needs B == 1 ...
    assert _bwd(lib, bias=3, B=1, ns=1) == INVALID         # ... and offsets
    assert _bwd(lib, K=32) == UNSUPPORTED
    assert _bwd(lib, dq=40) == UNSUPPORTED                 # 16-byte alignment
    assert _bwd(lib, ws=None) == WORKSPACE
    assert _bwd(lib, wsb=1024) == WORKSPACE
    assert _bwd(lib, ws=512 + 16) == WORKSPACE             # 256-byte alignment
    assert _bwd(lib, B=0) == 0
    assert _bwd(lib, M=0, N=0) == 0


def test_block_sparse_rejects_bad_arguments(lib):
    INVALID, UNSUPPORTED = -1, -2
    vp = ctypes.c_void_p

    def call(bias=0, mask=16, ms=(0, 0), K=64, scale=0.1):
        s = I64x3(1024, 64 * 4, 64)
        mst = (ctypes.c_int64 * 2)(*ms) if ms is not None else None
        return lib.mea_fwd_block_sparse(vp(16), vp(16), vp(16), vp(16), None, 1, 128, 128, 4, 4,
                                        K, s, s, s, s, 0, bias, vp(mask), mst, 0,
                                        ctypes.c_float(scale), None)
    assert lib.mea_sparse_block_size() == 128
    assert call(bias=2) == UNSUPPORTED
    assert call(bias=3) == UNSUPPORTED
    assert call(bias=7) == INVALID
    assert call(mask=None) == INVALID
    assert call(ms=(-1, 0)) == INVALID
    assert call(ms=None) == INVALID
    assert call(K=96) == UNSUPPORTED


def test_prefill_chunk_rejects_bad_arguments(lib):
    INVALID, UNSUPPORTED = -1, -2
    vp = ctypes.c_void_p

    def call(B=2, M=64, cap=128, Hq=4, Hkv=2, K=64, dtype=0, causal=1, scale=0.1, cl=16, kc=16,
             q=16):
        s = I64x3(1 << 20, 1024, 128)
        return lib.mea_prefill_chunk(vp(q), vp(16), vp(16), vp(kc), vp(16), vp(cl), None, vp(16),
                                     None, B, M, cap, Hq, Hkv, K, s, s, s, s, s, s, dtype, causal,
                                     0, ctypes.c_float(scale), None)
    assert call(Hq=3) == INVALID
    assert call(dtype=4) == INVALID
    assert call(causal=2) == INVALID
    assert call(cl=None) == INVALID
    assert call(kc=None) == INVALID
    assert call(cap=0) == INVALID
    assert call(scale=float("nan")) == INVALID
    assert call(K=80) == UNSUPPORTED
    assert call(scale=-1.0) == UNSUPPORTED
    assert call(q=8) == UNSUPPORTED
    assert call(B=0) == 0
    assert call(M=0) == 0


def test_bench_ex2_ceiling():
    """The secondary roofline of the bench line: 148 SMs x 16 ex2/clk x the SM
    clock x 256 FLOP per score (K = 64): 1191.2 TFLOP/s at the 1965 MHz maximum,
    1122.7 at a sampled 1852 MHz."""
    import bench

    r = bench.ex2_roofline(595.6, 148, 64)
    assert r["peak"] == 1191.2
    assert abs(r["frac"] - 0.5) < 1e-3  # 595.6 / 1191.2
    assert r["unit"] == "TFLOP/s"
    r = bench.ex2_roofline(561.35, 148, 64, sm_mhz=1852.0)
    assert r["peak"] == 1122.7
    assert abs(r["frac"] - 0.5) < 1e-3
