"""memory_efficient_exact_mea_b200 -- memory-efficient exact attention on B200.

A thin ctypes binding of ``libmea.so`` (C ABI in ``include/mea.h``).  This module
only marshals arguments: every step of the computation runs in the library's
sm_100a kernels.  PyTorch supplies device memory and the current stream.  There
is no fallback: importing this package fails loudly if ``libmea.so`` is missing.

Operations (sources cited in ``include/mea.h``):
  mea_fwd     softmax(Q K^T * scale + bias) V and the per-row log-sum-exp, with
              no / causal / block-diagonal (causal) masks, GQA and ALiBi.
  mea_fwd_block_sparse  mea_fwd with whole 128x128 score blocks left out by a mask.
  mea_prefill_chunk  a chunk of new queries against a KV cache, appending its keys/values.
  mea_bwd     dq, dk, dv by recomputing the weights from the forward's lse.
  mea_decode  one query per sequence against a packed, ragged KV cache.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["mea_fwd", "mea_fwd_block_sparse", "mea_prefill_chunk", "mea_bwd", "mea_decode",
           "mea_decode_workspace_size", "mea_decode_chunk", "read_device_status", "status_string",
           "MeaError", "PreparedCall", "BIAS", "BWD_PREP", "BWD_MAIN", "BWD_DQ", "LIB_PATH", "lib"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmea.so")

BIAS = {"none": 0, "causal": 1, "blockdiag": 2, "blockdiag_causal": 3}
BWD_PREP, BWD_MAIN, BWD_DQ = 1, 2, 4  # stages of the backward (mea_bwd_stages)
_DTYPE = {torch.float16: 0, torch.bfloat16: 1}
_i64x3 = ctypes.c_int64 * 3


class MeaError(RuntimeError):
    """A libmea entry point returned an error status."""

    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {status_string(code)} ({code})")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python memory_efficient_exact_mea_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.mea_fwd.restype = i
    L.mea_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, vp, vp, vp, i, i, vp, vp,
                          i, i, i, i, f, vp]
    L.mea_decode_workspace_size.restype = sz
    L.mea_decode_workspace_size.argtypes = [i, i, i, i, i]
    L.mea_decode.restype = i
    L.mea_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp, sz, vp]
    L.mea_fwd_block_sparse.restype = i
    L.mea_fwd_block_sparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, vp, vp, vp, i, i,
                                       vp, vp, i, f, vp]
    L.mea_prefill_chunk.restype = i
    L.mea_prefill_chunk.argtypes = [vp] * 9 + [i] * 6 + [vp] * 6 + [i, i, i, f, vp]
    L.mea_sparse_block_size.restype = i
    L.mea_sparse_block_size.argtypes = []
    L.mea_bwd_workspace_size.restype = sz
    L.mea_bwd_workspace_size.argtypes = [i, i, i, i]
    L.mea_bwd.restype = i
    L.mea_bwd.argtypes = [vp] * 9 + [i] * 8 + [vp, vp, i, i, i, i, f, vp, sz, vp]
    L.mea_bwd_stages.restype = i
    L.mea_bwd_stages.argtypes = [vp] * 9 + [i] * 8 + [vp, vp, i, i, i, i, f, vp, sz, i, vp]
    L.mea_decode_chunk.restype = i
    L.mea_decode_chunk.argtypes = []
    L.mea_status_string.restype = ctypes.c_char_p
    L.mea_status_string.argtypes = [i]
    L.mea_read_device_status.restype = i
    L.mea_read_device_status.argtypes = [vp, i]
    L.mea_version.restype = i
    L.mea_version.argtypes = []
    return L


lib = _load()


def status_string(code: int) -> str:
    return lib.mea_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, device=None):
    """The CUDA stream handle to launch on: `stream`, else the current stream of
    `device` (a torch.device, default the current device)."""
    if stream is None:
        if _raw_stream is not None and device is not None and device.index is not None:
            return ctypes.c_void_p(_raw_stream(device.index))
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise MeaError(fn, rc)


_STRIDES: dict = {}  # (sb, sm, sh) -> ctypes int64[3], reused across calls (read-only)



def _bmhk_strides(t: torch.Tensor, name: str):
    st = t.stride()
    if len(st) != 4:
        raise ValueError(f"{name} must be [B, rows, heads, K]")
    if st[3] != 1:
        raise ValueError(f"{name}: the last dimension must be contiguous")
    key = st[:3]
    arr = _STRIDES.get(key)
    if arr is None:
        if len(_STRIDES) > 4096:
            _STRIDES.clear()
        arr = _STRIDES[key] = _i64x3(*key)
    return arr


def _grouped_views(q, k, v, out):
    """The 5-D grouped-query layout as 4-D views (no copy): q [B,M,G,H,K] ->
    [B,M,G*H,K] (query head g*H + r); k, v [B,N,G,1,K], or [B,N,G,H,K] expanded
    along H with stride 0, -> [B,N,G,K] (key/value head g, shared by the H query
    heads of group g); k, v with a real H axis -> [B,N,G*H,K]."""
    B, M, G, H, K = q.shape
    if k.dim() != 5 or v.dim() != 5 or k.shape[:3] != v.shape[:3] or k.shape[2] != G:
        raise ValueError("5-D q [B,M,G,H,K] needs k, v [B,N,G,1|H,K]")

    def flat(t, name):
        if t.shape[3] != 1 and t.stride(2) != t.shape[3] * t.stride(3):
            raise ValueError(f"{name}: the group and head axes must merge into one (a view)")
        return t.flatten(2, 3)

    def kv4(t, name):
        if t.shape[3] == 1 or t.stride(3) == 0:
            return t[:, :, :, 0]
        return flat(t, name)

    q4 = flat(q, "q")
    o4 = None if out is None else flat(out, "out")
    return q4, kv4(k, "k"), kv4(v, "v"), o4


class PreparedCall:
    """One C-ABI call with every argument marshalled once, for launching the same
    computation again and again (a serving or training loop whose buffers stay
    put): calling it only runs the C entry point, on the stream chosen when it
    was prepared.  It keeps the tensors it points into alive.  `outputs` holds
    what the call writes."""

    __slots__ = ("_fn", "_args", "_name", "_keep", "outputs")

    def __init__(self, fn, args, name, keep, outputs):
        self._fn, self._args, self._name, self._keep, self.outputs = fn, args, name, keep, outputs

    def __call__(self):
        rc = self._fn(*self._args)
        if rc != 0:
            raise MeaError(self._name, rc)
        return self.outputs


def mea_fwd(q, k, v, bias: str = "none", scale: float | None = None, alibi: bool = False,
            seqstart_q=None, seqstart_k=None, max_seqlen_q: int | None = None,
            max_seqlen_k: int | None = None, out=None, lse=None, return_lse: bool = True,
            stream=None, prepare: bool = False):
    """Attention forward.  q [B,M,Hq,K], k/v [B,N,Hkv,K] (fp16/bf16, CUDA) ->
    (out [B,M,Hq,K], lse [B,Hq,M] fp32 or None).

    bias: "none" | "causal" | "blockdiag" | "blockdiag_causal".  The block-diagonal
    kinds take B == 1 and int32 CUDA offsets ``seqstart_q`` (and ``seqstart_k``);
    ``max_seqlen_q`` is the longest query sequence (read from the offsets, with a
    device-to-host copy, when not given).

    Grouped-query 5-D layout: q [B,M,G,H,K] with k, v [B,N,G,1,K] (or expanded to
    [B,N,G,H,K] with stride 0) is the same call with Hq = G*H query heads and
    Hkv = G key/value heads, query head g*H + r reading key/value head g; out is
    returned as [B,M,G,H,K] and lse as [B,G*H,M].

    prepare=True launches nothing and returns a PreparedCall instead: each call
    of it runs this forward again on the same buffers (its outputs are
    (out, lse)), with no Python-side argument handling.
    """
    if q.dim() == 5:
        if prepare:
            raise ValueError("prepare=True takes the 4-D layout")
        shape5 = tuple(q.shape)
        q, k, v, out4 = _grouped_views(q, k, v, out)
        o, l = mea_fwd(q, k, v, bias, scale, alibi, seqstart_q, seqstart_k, max_seqlen_q,
                       max_seqlen_k, out4, lse, return_lse, stream)
        return o.view(shape5) if out is None else out, l
    B, M, Hq, K = q.shape
    N, Hkv = k.shape[1], k.shape[2]
    if q.dtype not in _DTYPE or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype float16 or bfloat16")
    if tuple(k.shape) != (B, N, Hkv, K) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, N, Hkv, K]")
    scale = K ** -0.5 if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, M, Hq, K), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, M), dtype=torch.float32, device=q.device)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 [B, Hq, M] tensor")
    kind = BIAS[bias]
    ns = 0
    if kind >= 2:
        if seqstart_q is None:
            raise ValueError("block-diagonal bias needs seqstart_q")
        for s in (seqstart_q, seqstart_k):
            if s is not None and (s.dtype != torch.int32 or not s.is_cuda):
                raise ValueError("seqstart offsets must be int32 CUDA tensors")
        ns = seqstart_q.numel() - 1
        if max_seqlen_q is None:
            max_seqlen_q = int(torch.diff(seqstart_q).max().item()) if ns > 0 else 0
        if max_seqlen_k is None:
            sk = seqstart_q if seqstart_k is None else seqstart_k
            max_seqlen_k = int(torch.diff(sk).max().item()) if ns > 0 else 0
    else:
        seqstart_q = seqstart_k = None
        max_seqlen_q = max_seqlen_k = 0
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, M, N, Hq, Hkv, K,
            _bmhk_strides(q, "q"), _bmhk_strides(k, "k"), _bmhk_strides(v, "v"),
            _bmhk_strides(out, "out"), _DTYPE[q.dtype], kind, _ptr(seqstart_q), _ptr(seqstart_k),
            ns, int(max_seqlen_q), int(max_seqlen_k), int(bool(alibi)), scale,
            _stream(stream, q.device))
    if prepare:
        return PreparedCall(lib.mea_fwd, args, "mea_fwd",
                            (q, k, v, out, lse, seqstart_q, seqstart_k), (out, lse))
    _check("mea_fwd", lib.mea_fwd(*args))
    return out, lse


def mea_fwd_block_sparse(q, k, v, block_mask, bias: str = "none", scale: float | None = None,
                         alibi: bool = False, out=None, lse=None, return_lse: bool = True,
                         stream=None):
    """Block-sparse attention forward.  As ``mea_fwd`` (bias "none" or "causal"),
    plus ``block_mask``: a uint8 CUDA tensor [B, Hq, ceil(M/128), ceil(N/128)]
    (size-1 or stride-0 batch/head dimensions broadcast; the last two dimensions
    contiguous); a zero entry leaves that 128x128 block of scores out."""
    B, M, Hq, K = q.shape
    N, Hkv = k.shape[1], k.shape[2]
    if q.dtype not in _DTYPE or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype float16 or bfloat16")
    if tuple(k.shape) != (B, N, Hkv, K) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, N, Hkv, K]")
    blk = int(lib.mea_sparse_block_size())
    mb, nb = -(-M // blk), -(-N // blk)
    if (block_mask.dtype != torch.uint8 or block_mask.dim() != 4 or not block_mask.is_cuda
            or tuple(block_mask.shape[2:]) != (mb, nb)
            or block_mask.shape[0] not in (1, B) or block_mask.shape[1] not in (1, Hq)):
        raise ValueError(f"block_mask must be a uint8 CUDA tensor [B|1, Hq|1, {mb}, {nb}]")
    if block_mask.stride(3) != 1 or block_mask.stride(2) != nb:
        raise ValueError("block_mask: the last two dimensions must be contiguous")
    mst = (ctypes.c_int64 * 2)(block_mask.stride(0) if block_mask.shape[0] > 1 else 0,
                               block_mask.stride(1) if block_mask.shape[1] > 1 else 0)
    scale = K ** -0.5 if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, M, Hq, K), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, M), dtype=torch.float32, device=q.device)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 [B, Hq, M] tensor")
    rc = lib.mea_fwd_block_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, M, N, Hq,
                                  Hkv, K, _bmhk_strides(q, "q"), _bmhk_strides(k, "k"),
                                  _bmhk_strides(v, "v"), _bmhk_strides(out, "out"),
                                  _DTYPE[q.dtype], BIAS[bias], _ptr(block_mask), mst,
                                  int(bool(alibi)), scale, _stream(stream, q.device))
    _check("mea_fwd_block_sparse", rc)
    return out, lse


def mea_prefill_chunk(q, k_new, v_new, k_cache, v_cache, cache_seqlens, q_seqlens=None,
                      causal: bool = True, scale: float | None = None, alibi: bool = False,
                      out=None, lse=None, return_lse: bool = True, stream=None):
    """One prefill chunk against a KV cache, with the append fused in.

    q [B,M,Hq,K], k_new/v_new [B,M,Hkv,K], k_cache/v_cache [B,cap,Hkv,K] (updated
    in place: rows cache_seqlens[b] .. + q_seqlens[b] receive the chunk's keys and
    values), cache_seqlens / q_seqlens int32 CUDA [B] (q_seqlens None: every
    sequence has M new rows).  Returns (out [B,M,Hq,K], lse [B,Hq,M] or None);
    rows past q_seqlens[b] are not written.  The caller advances cache_seqlens."""
    B, M, Hq, K = q.shape
    cap, Hkv = k_cache.shape[1], k_cache.shape[2]
    ts = (q, k_new, v_new, k_cache, v_cache)
    if q.dtype not in _DTYPE or any(t.dtype != q.dtype for t in ts):
        raise ValueError("q, k_new, v_new, k_cache, v_cache must share dtype float16 or bfloat16")
    if tuple(k_new.shape) != (B, M, Hkv, K) or tuple(v_new.shape) != (B, M, Hkv, K):
        raise ValueError("k_new and v_new must be [B, M, Hkv, K]")
    if tuple(k_cache.shape) != (B, cap, Hkv, K) or tuple(v_cache.shape) != (B, cap, Hkv, K):
        raise ValueError("k_cache and v_cache must be [B, cap, Hkv, K]")
    for name, t in (("cache_seqlens", cache_seqlens), ("q_seqlens", q_seqlens)):
        if t is not None and (t.dtype != torch.int32 or not t.is_cuda or t.numel() != B):
            raise ValueError(f"{name} must be an int32 CUDA tensor of B entries")
    scale = K ** -0.5 if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, M, Hq, K), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, M), dtype=torch.float32, device=q.device)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 [B, Hq, M] tensor")
    rc = lib.mea_prefill_chunk(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                               _ptr(cache_seqlens), _ptr(q_seqlens), _ptr(out), _ptr(lse), B, M,
                               cap, Hq, Hkv, K, _bmhk_strides(q, "q"),
                               _bmhk_strides(k_new, "k_new"), _bmhk_strides(v_new, "v_new"),
                               _bmhk_strides(k_cache, "k_cache"),
                               _bmhk_strides(v_cache, "v_cache"), _bmhk_strides(out, "out"),
                               _DTYPE[q.dtype], int(bool(causal)), int(bool(alibi)), scale,
                               _stream(stream, q.device))
    _check("mea_prefill_chunk", rc)
    return out, lse


def mea_bwd(q, k, v, out, dout, lse, bias: str = "none", scale: float | None = None,
            alibi: bool = False, seqstart_q=None, seqstart_k=None,
            max_seqlen_q: int | None = None, max_seqlen_k: int | None = None,
            dq=None, dk=None, dv=None, workspace=None, stages: int = 7, stream=None):
    """Attention backward.  Contiguous q/out/dout [B,M,Hq,K], k/v [B,N,Hkv,K] and the
    forward's lse [B,Hq,M] -> (dq, dk, dv) shaped like q, k, v.

    ``stages`` (bitwise OR of BWD_PREP, BWD_MAIN, BWD_DQ; default all) runs only
    those launches of the backward (mea_bwd_stages); running them one at a time
    with the same arguments and workspace equals one full call."""
    B, M, Hq, K = q.shape
    N, Hkv = k.shape[1], k.shape[2]
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dtype not in _DTYPE or any(t.dtype != q.dtype for t in (k, v, out, dout)):
        raise ValueError("q, k, v, out, dout must share dtype float16 or bfloat16")
    scale = K ** -0.5 if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = int(lib.mea_bwd_workspace_size(B, M, Hq, K))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    kind = BIAS[bias]
    ns = 0
    if kind >= 2:
        ns = seqstart_q.numel() - 1
        if max_seqlen_q is None:
            max_seqlen_q = int(torch.diff(seqstart_q).max().item()) if ns > 0 else 0
        if max_seqlen_k is None:
            sk = seqstart_q if seqstart_k is None else seqstart_k
            max_seqlen_k = int(torch.diff(sk).max().item()) if ns > 0 else 0
    else:
        seqstart_q = seqstart_k = None
        max_seqlen_q = max_seqlen_k = 0
    rc = lib.mea_bwd_stages(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                            _ptr(dq), _ptr(dk), _ptr(dv), B, M, N, Hq, Hkv, K, _DTYPE[q.dtype],
                            kind, _ptr(seqstart_q), _ptr(seqstart_k), ns, int(max_seqlen_q),
                            int(max_seqlen_k), int(bool(alibi)), scale, _ptr(workspace), ws_bytes,
                            int(stages), _stream(stream, q.device))
    _check("mea_bwd", rc)
    return dq, dk, dv


def mea_decode_workspace_size(B: int, Hq: int, Hkv: int, K: int, max_kv_len: int) -> int:
    return int(lib.mea_decode_workspace_size(B, Hq, Hkv, K, max_kv_len))


def mea_decode_chunk() -> int:
    return int(lib.mea_decode_chunk())


def mea_decode(q, k_cache, v_cache, kv_seqstart, max_kv_len: int, scale: float | None = None,
               alibi: bool = False, out=None, lse=None, workspace=None, return_lse: bool = True,
               stream=None):
    """One decode step.  q [B,Hq,K] or [B,1,Hq,K]; caches [T,Hkv,K]; kv_seqstart int32
    CUDA [B+1] -> (out shaped like q, lse [B,Hq] fp32 or None)."""
    qshape = tuple(q.shape)
    q3 = q.reshape(q.shape[0], q.shape[-2], q.shape[-1])
    B, Hq, K = q3.shape
    T, Hkv = k_cache.shape[0], k_cache.shape[1]
    for name, t in (("q", q3), ("k_cache", k_cache), ("v_cache", v_cache)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if tuple(v_cache.shape) != tuple(k_cache.shape) or k_cache.shape[2] != K:
        raise ValueError("caches must be [T, Hkv, K]")
    if q.dtype not in _DTYPE or k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("q and caches must share dtype float16 or bfloat16")
    if kv_seqstart.dtype != torch.int32 or not kv_seqstart.is_cuda:
        raise ValueError("kv_seqstart must be an int32 CUDA tensor")
    scale = K ** -0.5 if scale is None else float(scale)
    if out is None:
        out = torch.empty(qshape, dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = mea_decode_workspace_size(B, Hq, Hkv, K, max_kv_len)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.mea_decode(_ptr(q3), _ptr(k_cache), _ptr(v_cache), _ptr(kv_seqstart), _ptr(out),
                        _ptr(lse), B, Hq, Hkv, K, T, int(max_kv_len), _DTYPE[q.dtype],
                        int(bool(alibi)), scale, _ptr(workspace), ws_bytes, _stream(stream, q.device))
    _check("mea_decode", rc)
    return out, lse


def read_device_status(clear: bool = True, stream=None) -> int:
    """Synchronise and return the first error a kernel recorded on this device (0 = none)."""
    return int(lib.mea_read_device_status(_stream(stream), int(bool(clear))))
