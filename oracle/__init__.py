"""fp64 CPU oracle for memory-efficient exact attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path.
The arithmetic lives in ``mea_oracle.c`` (plain C, fp64, one query row at a
time); this module only marshals arrays through ctypes.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, invariants, brute force) and the pins are themselves checked
against planted mistakes by ``tests/test_oracle_mutants.py``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, default_library_path

BIAS_NONE, BIAS_CAUSAL, BIAS_BLOCKDIAG, BIAS_BLOCKDIAG_CAUSAL = 0, 1, 2, 3

_c_double_p = ctypes.POINTER(ctypes.c_double)
_c_int32_p = ctypes.POINTER(ctypes.c_int32)
_c_int64_p = ctypes.POINTER(ctypes.c_int64)
_c_uint8_p = ctypes.POINTER(ctypes.c_uint8)


def _f64(x) -> np.ndarray:
    """Exact conversion to a contiguous float64 array (fp16/bf16 -> fp64 is exact)."""
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch

        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray | None:
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a, typ):
    return None if a is None else a.ctypes.data_as(typ)


class Oracle:
    """ctypes handle on one build of the oracle library."""

    def __init__(self, path: str | None = None):
        path = path or default_library_path()
        if not os.path.exists(path):
            build_oracle(out=path)
        lib = ctypes.CDLL(path)
        lib.oracle_alibi_slope.restype = ctypes.c_double
        lib.oracle_alibi_slope.argtypes = [ctypes.c_int, ctypes.c_int]
        lib.oracle_alibi_slopes.restype = None
        lib.oracle_alibi_slopes.argtypes = [ctypes.c_int, _c_double_p]
        common = [_c_double_p, _c_double_p, _c_double_p] + [ctypes.c_int] * 7 + [
            _c_int32_p, _c_int32_p, ctypes.c_int, _c_double_p, ctypes.c_double]
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = common + [_c_double_p, _c_double_p]
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_attention_rows.argtypes = common + [_c_int64_p, ctypes.c_int64,
                                                       _c_double_p, _c_double_p]
        lib.oracle_attention_bwd.restype = ctypes.c_int
        lib.oracle_attention_bwd.argtypes = [_c_double_p] * 4 + [ctypes.c_int] * 7 + [
            _c_int32_p, _c_int32_p, ctypes.c_int, _c_double_p, ctypes.c_double,
            _c_double_p, _c_double_p, _c_double_p]
        lib.oracle_attention_block_sparse.restype = ctypes.c_int
        lib.oracle_attention_block_sparse.argtypes = [_c_double_p] * 3 + [ctypes.c_int] * 7 + [
            _c_uint8_p, ctypes.c_int, ctypes.c_int, _c_double_p, ctypes.c_double, _c_int64_p,
            ctypes.c_int64, _c_double_p, _c_double_p]
        lib.oracle_prefill_chunk.restype = ctypes.c_int
        lib.oracle_prefill_chunk.argtypes = [_c_double_p] * 5 + [_c_int32_p, _c_int32_p] + [
            ctypes.c_int] * 7 + [_c_double_p, ctypes.c_double, _c_double_p, _c_double_p]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [_c_double_p, _c_double_p, _c_double_p, _c_int32_p,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      _c_double_p, ctypes.c_double, _c_double_p, _c_double_p]
        self.lib = lib
        self.path = path

    # -- ALiBi ---------------------------------------------------------------
    def alibi_slopes(self, Hq: int) -> np.ndarray:
        """Slopes 2^(-8(h+1)/Hq) for query heads h = 0..Hq-1."""
        s = np.zeros(Hq, dtype=np.float64)
        self.lib.oracle_alibi_slopes(Hq, _ptr(s, _c_double_p))
        return s

    def _slopes(self, alibi, Hq):
        if alibi is None or alibi is False:
            return None
        if alibi is True:
            return self.alibi_slopes(Hq)
        s = _f64(alibi)
        assert s.shape == (Hq,)
        return s

    # -- prefill -------------------------------------------------------------
    def attention(self, q, k, v, bias=BIAS_NONE, scale=None, alibi=None,
                  seqstart_q=None, seqstart_k=None):
        """Full attention.  q [B,M,Hq,D], k/v [B,N,Hkv,D] -> (out [B,M,Hq,D], lse [B,Hq,M]).

        ``alibi`` is None/False, True (standard slopes) or an explicit slope array.
        """
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, M, Hq, D = q.shape
        N, Hkv = k.shape[1], k.shape[2]
        assert k.shape == (B, N, Hkv, D) and v.shape == k.shape
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        sq, sk = _i32(seqstart_q), _i32(seqstart_k)
        if sk is None:
            sk = sq
        ns = 0 if sq is None else len(sq) - 1
        slopes = self._slopes(alibi, Hq)
        out = np.zeros((B, M, Hq, D), dtype=np.float64)
        lse = np.zeros((B, Hq, M), dtype=np.float64)
        rc = self.lib.oracle_attention(
            _ptr(q, _c_double_p), _ptr(k, _c_double_p), _ptr(v, _c_double_p),
            B, M, N, Hq, Hkv, D, int(bias), _ptr(sq, _c_int32_p), _ptr(sk, _c_int32_p), ns,
            _ptr(slopes, _c_double_p), scale, _ptr(out, _c_double_p), _ptr(lse, _c_double_p))
        if rc != 0:
            raise ValueError("oracle_attention rejected its arguments")
        return out, lse

    def attention_rows(self, q, k, v, rows, bias=BIAS_NONE, scale=None, alibi=None,
                       seqstart_q=None, seqstart_k=None):
        """Selected rows.  rows: int array [n, 3] of (b, i, h) -> (out [n, D], lse [n])."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, M, Hq, D = q.shape
        N, Hkv = k.shape[1], k.shape[2]
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        sq, sk = _i32(seqstart_q), _i32(seqstart_k)
        if sk is None:
            sk = sq
        ns = 0 if sq is None else len(sq) - 1
        slopes = self._slopes(alibi, Hq)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = rows.shape[0]
        out = np.zeros((n, D), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        rc = self.lib.oracle_attention_rows(
            _ptr(q, _c_double_p), _ptr(k, _c_double_p), _ptr(v, _c_double_p),
            B, M, N, Hq, Hkv, D, int(bias), _ptr(sq, _c_int32_p), _ptr(sk, _c_int32_p), ns,
            _ptr(slopes, _c_double_p), scale, _ptr(rows, _c_int64_p), n,
            _ptr(out, _c_double_p), _ptr(lse, _c_double_p))
        if rc != 0:
            raise ValueError("oracle_attention_rows rejected its arguments")
        return out, lse

    def attention_bwd(self, q, k, v, dout, bias=BIAS_NONE, scale=None, alibi=None,
                      seqstart_q=None, seqstart_k=None):
        """Gradients of sum(out * dout) -> (dq [B,M,Hq,D], dk, dv [B,N,Hkv,D])."""
        q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, M, Hq, D = q.shape
        N, Hkv = k.shape[1], k.shape[2]
        assert do.shape == q.shape
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        sq, sk = _i32(seqstart_q), _i32(seqstart_k)
        if sk is None:
            sk = sq
        ns = 0 if sq is None else len(sq) - 1
        slopes = self._slopes(alibi, Hq)
        dq = np.zeros_like(q)
        dk = np.zeros_like(k)
        dv = np.zeros_like(v)
        rc = self.lib.oracle_attention_bwd(
            _ptr(q, _c_double_p), _ptr(k, _c_double_p), _ptr(v, _c_double_p),
            _ptr(do, _c_double_p), B, M, N, Hq, Hkv, D, int(bias), _ptr(sq, _c_int32_p),
            _ptr(sk, _c_int32_p), ns, _ptr(slopes, _c_double_p), scale,
            _ptr(dq, _c_double_p), _ptr(dk, _c_double_p), _ptr(dv, _c_double_p))
        if rc != 0:
            raise ValueError("oracle_attention_bwd rejected its arguments")
        return dq, dk, dv

    def attention_block_sparse(self, q, k, v, block_mask, block_m, block_n, bias=BIAS_NONE,
                               scale=None, alibi=None, rows=None):
        """Block-sparse attention.  block_mask: uint8 [B, Hq, ceil(M/block_m),
        ceil(N/block_n)] (0 = block left out).  rows None -> (out [B,M,Hq,D],
        lse [B,Hq,M]); rows int [n, 3] of (b, i, h) -> (out [n, D], lse [n])."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, M, Hq, D = q.shape
        N, Hkv = k.shape[1], k.shape[2]
        assert k.shape == (B, N, Hkv, D) and v.shape == k.shape
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        mask = block_mask
        if hasattr(mask, "detach"):
            mask = mask.detach().to("cpu").numpy()
        mask = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
        mb, nb = -(-M // block_m), -(-N // block_n)
        assert mask.shape == (B, Hq, mb, nb), (mask.shape, (B, Hq, mb, nb))
        slopes = self._slopes(alibi, Hq)
        if rows is None:
            out = np.zeros((B, M, Hq, D), dtype=np.float64)
            lse = np.zeros((B, Hq, M), dtype=np.float64)
            rows_p, n = None, 0
        else:
            rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
            n = rows.shape[0]
            out = np.zeros((n, D), dtype=np.float64)
            lse = np.zeros((n,), dtype=np.float64)
            rows_p = _ptr(rows, _c_int64_p)
        rc = self.lib.oracle_attention_block_sparse(
            _ptr(q, _c_double_p), _ptr(k, _c_double_p), _ptr(v, _c_double_p),
            B, M, N, Hq, Hkv, D, int(bias), _ptr(mask, _c_uint8_p), int(block_m), int(block_n),
            _ptr(slopes, _c_double_p), scale, rows_p, n,
            _ptr(out, _c_double_p), _ptr(lse, _c_double_p))
        if rc != 0:
            raise ValueError("oracle_attention_block_sparse rejected its arguments")
        return out, lse

    def prefill_chunk(self, q, k_new, v_new, k_cache, v_cache, cache_len, q_len=None,
                      causal=True, scale=None, alibi=None):
        """One prefill chunk against a cache.  q [B,M,Hq,D], k_new/v_new [B,M,Hkv,D],
        caches [B,cap,Hkv,D], cache_len [B] (rows already cached), q_len [B] or None
        (= M) -> (out [B,M,Hq,D], lse [B,Hq,M], k_cache', v_cache').  Rows i >= q_len[b]
        of out are 0 and of lse are nan (not computed)."""
        q, kn, vn = _f64(q), _f64(k_new), _f64(v_new)
        kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
        B, M, Hq, D = q.shape
        cap, Hkv = kc.shape[1], kc.shape[2]
        assert kn.shape == (B, M, Hkv, D) and vn.shape == kn.shape
        assert kc.shape == (B, cap, Hkv, D) and vc.shape == kc.shape
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        cl = _i32(cache_len)
        ql = _i32(q_len)
        slopes = self._slopes(alibi, Hq)
        out = np.zeros((B, M, Hq, D), dtype=np.float64)
        lse = np.full((B, Hq, M), np.nan, dtype=np.float64)
        rc = self.lib.oracle_prefill_chunk(
            _ptr(q, _c_double_p), _ptr(kn, _c_double_p), _ptr(vn, _c_double_p),
            _ptr(kc, _c_double_p), _ptr(vc, _c_double_p), _ptr(cl, _c_int32_p),
            _ptr(ql, _c_int32_p), B, M, cap, Hq, Hkv, D, int(bool(causal)),
            _ptr(slopes, _c_double_p), scale, _ptr(out, _c_double_p), _ptr(lse, _c_double_p))
        if rc != 0:
            raise ValueError("oracle_prefill_chunk rejected its arguments")
        return out, lse, kc, vc

    # -- decode --------------------------------------------------------------
    def decode(self, q, k_cache, v_cache, kv_seqstart, scale=None, alibi=None):
        """One decode step.  q [B,Hq,D] (or [B,1,Hq,D]), caches [T,Hkv,D] ->
        (out [B,Hq,D], lse [B,Hq])."""
        q = _f64(q)
        if q.ndim == 4:
            q = np.ascontiguousarray(q[:, 0])
        kc, vc = _f64(k_cache), _f64(v_cache)
        B, Hq, D = q.shape
        Hkv = kc.shape[1]
        st = _i32(kv_seqstart)
        assert st.shape == (B + 1,)
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        slopes = self._slopes(alibi, Hq)
        out = np.zeros((B, Hq, D), dtype=np.float64)
        lse = np.zeros((B, Hq), dtype=np.float64)
        rc = self.lib.oracle_decode(
            _ptr(q, _c_double_p), _ptr(kc, _c_double_p), _ptr(vc, _c_double_p),
            _ptr(st, _c_int32_p), B, Hq, Hkv, D, _ptr(slopes, _c_double_p), scale,
            _ptr(out, _c_double_p), _ptr(lse, _c_double_p))
        if rc != 0:
            raise ValueError("oracle_decode rejected its arguments")
        return out, lse


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from this directory's source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
