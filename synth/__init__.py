"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CUDA path and the oracle can consume its
output without sharing any of the method.

Recipe: a CPU ``torch.Generator`` seeded per workload, ``randn`` in float32,
then a cast to the workload dtype (fp16 or bf16).  Packed-sequence lengths come
from ``torch.randint`` on the same kind of generator (inclusive bounds).  The
shapes mirror the workloads of the pages (xFormers tutorial: B, M, H, K = 2,
256, 8, 64 with a lower-triangular mask; a 512..4096 sequence sweep; packed
variable-length batches; grouped-query heads with ALiBi; a KV-cache decode
step).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn(shape, dtype: str, g: torch.Generator) -> torch.Tensor:
    """N(0,1) float32 draws cast to fp16/bf16 (CPU, contiguous)."""
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(DTYPES[dtype])


def lengths(n: int, lo: int, hi: int, g: torch.Generator) -> torch.Tensor:
    """n integer lengths drawn uniformly from [lo, hi] inclusive (int32)."""
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64).to(torch.int32)


def offsets(lens) -> torch.Tensor:
    """Start offsets [0, l0, l0+l1, ...] (int32, len(lens)+1) of a packed batch."""
    lens = torch.as_tensor(lens, dtype=torch.int64)
    out = torch.zeros(len(lens) + 1, dtype=torch.int64)
    out[1:] = torch.cumsum(lens, 0)
    return out.to(torch.int32)


@dataclass
class Prefill:
    """One prefill problem: q [B,M,Hq,K], k/v [B,N,Hkv,K] (CPU tensors)."""

    name: str
    B: int
    M: int
    N: int
    Hq: int
    Hkv: int
    K: int
    dtype: str
    bias: str  # "none" | "causal" | "blockdiag" | "blockdiag_causal"
    alibi: bool = False
    seed: int = 0
    seq_lens_q: list | None = None
    seq_lens_k: list | None = None
    q: torch.Tensor | None = field(default=None, repr=False)
    k: torch.Tensor | None = field(default=None, repr=False)
    v: torch.Tensor | None = field(default=None, repr=False)

    @property
    def seqstart_q(self):
        return None if self.seq_lens_q is None else offsets(self.seq_lens_q)

    @property
    def seqstart_k(self):
        lens = self.seq_lens_k if self.seq_lens_k is not None else self.seq_lens_q
        return None if lens is None else offsets(lens)

    @property
    def scale(self) -> float:
        return float(self.K) ** -0.5


@dataclass
class Decode:
    """One decode step: q [B,1,Hq,K]; packed caches [T,Hkv,K]; kv_seqstart [B+1]."""

    name: str
    B: int
    Hq: int
    Hkv: int
    K: int
    dtype: str
    seed: int
    kv_lens: list
    alibi: bool = False
    q: torch.Tensor | None = field(default=None, repr=False)
    k_cache: torch.Tensor | None = field(default=None, repr=False)
    v_cache: torch.Tensor | None = field(default=None, repr=False)

    @property
    def kv_seqstart(self):
        return offsets(self.kv_lens)

    @property
    def max_kv_len(self) -> int:
        return int(max(self.kv_lens)) if len(self.kv_lens) else 0

    @property
    def scale(self) -> float:
        return float(self.K) ** -0.5


def make_prefill(name, B, M, N, Hq, Hkv, K, dtype, bias, alibi=False, seed=0,
                 seq_lens_q=None, seq_lens_k=None) -> Prefill:
    g = generator(seed)
    p = Prefill(name, B, M, N, Hq, Hkv, K, dtype, bias, alibi, seed,
                None if seq_lens_q is None else [int(x) for x in seq_lens_q],
                None if seq_lens_k is None else [int(x) for x in seq_lens_k])
    p.q = randn((B, M, Hq, K), dtype, g)
    p.k = randn((B, N, Hkv, K), dtype, g)
    p.v = randn((B, N, Hkv, K), dtype, g)
    return p


def make_varlen(name, lens_q, Hq, Hkv, K, dtype, causal, seed, lens_k=None, alibi=False):
    lens_k = lens_q if lens_k is None else lens_k
    M, N = int(sum(lens_q)), int(sum(lens_k))
    return make_prefill(name, 1, M, N, Hq, Hkv, K, dtype,
                        "blockdiag_causal" if causal else "blockdiag", alibi, seed,
                        list(lens_q), None if lens_k is lens_q else list(lens_k))


def make_decode(name, kv_lens, Hq, Hkv, K, dtype, seed, alibi=False) -> Decode:
    g = generator(seed + 7919)
    kv_lens = [int(x) for x in kv_lens]
    d = Decode(name, len(kv_lens), Hq, Hkv, K, dtype, seed, kv_lens, alibi)
    T = int(sum(kv_lens))
    d.q = randn((d.B, 1, Hq, K), dtype, g)
    d.k_cache = randn((T, Hkv, K), dtype, g)
    d.v_cache = randn((T, Hkv, K), dtype, g)
    return d


# ---------------------------------------------------------------------------
# The five workloads.  Seeds are 1000 + workload number.
# ---------------------------------------------------------------------------
SWEEP_M = (512, 1024, 2048, 4096)


def causal_small() -> Prefill:
    """Causal B=2, M=N=256, H=8, K=64, fp16, scale 1/8 (the tutorial's causal example)."""
    return make_prefill("causal_b2_m256_h8_k64_f16", 2, 256, 256, 8, 8, 64, "f16", "causal",
                        seed=1001)


def noncausal_sweep(M: int) -> Prefill:
    """Non-causal B=8, H=16, K=64, fp16, M=N in 512..4096 (the tutorial's sweep)."""
    return make_prefill(f"noncausal_b8_h16_k64_f16_m{M}", 8, M, M, 16, 16, 64, "f16", "none",
                        seed=1002 + M)


def varlen_lengths(n=32, lo=64, hi=2048, seed=1003):
    return lengths(n, lo, hi, generator(seed)).tolist()


def varlen_causal() -> Prefill:
    """32 packed sequences, lengths U[64, 2048], B=1, H=16, K=128, bf16, block-diagonal causal."""
    lens = varlen_lengths()
    return make_varlen("varlen32_causal_h16_k128_bf16", lens, 16, 16, 128, "bf16", True,
                       seed=1003)


def gqa_alibi_causal(M: int = 4096, B: int = 4) -> Prefill:
    """GQA + ALiBi causal: B=4, M=N=4096, Hq=32, Hkv=8, K=128, bf16."""
    return make_prefill(f"gqa_alibi_causal_b{B}_m{M}_hq32_hkv8_k128_bf16", B, M, M, 32, 8, 128,
                        "bf16", "causal", alibi=True, seed=1004)


def decode_lengths(n=64, lo=512, hi=8192, seed=1005):
    return lengths(n, lo, hi, generator(seed)).tolist()


def decode_step() -> Decode:
    """Decode: B=64, cached lengths U[512, 8192], Hq=32, Hkv=8, K=128, bf16 cache."""
    return make_decode("decode_b64_kv512-8192_hq32_hkv8_k128_bf16", decode_lengths(), 32, 8, 128,
                       "bf16", seed=1005)


def block_mask(B: int, Hq: int, M: int, N: int, block: int, density: float, seed: int,
               keep_diagonal: bool = False) -> torch.Tensor:
    """uint8 [B, Hq, ceil(M/block), ceil(N/block)]: each block kept (1) with
    probability `density` (independent uniform draws); with keep_diagonal the
    blocks (i, i) are always kept."""
    mb, nb = -(-M // block), -(-N // block)
    u = torch.rand((B, Hq, mb, nb), generator=generator(seed), dtype=torch.float32)
    m = (u < density).to(torch.uint8)
    if keep_diagonal:
        d = torch.arange(min(mb, nb))
        m[:, :, d, d] = 1
    return m


def block_sparse_noncausal(M: int = 4096) -> tuple[Prefill, torch.Tensor]:
    """Block-sparse non-causal: the sweep's B=8, H=16, K=64, fp16 at M=N, with 128x128
    blocks kept with probability 1/2 per (batch, head), diagonal blocks always kept."""
    p = make_prefill(f"block_sparse_b8_h16_k64_f16_m{M}_d50", 8, M, M, 16, 16, 64, "f16", "none",
                     seed=1006)
    return p, block_mask(8, 16, M, M, 128, 0.5, seed=1007, keep_diagonal=True)


@dataclass
class Chunk:
    """One prefill chunk against a KV cache: q [B,M,Hq,K], new k/v [B,M,Hkv,K],
    caches [B,cap,Hkv,K] holding past[b] rows, q_lens[b] real rows per chunk."""

    name: str
    B: int
    M: int
    cap: int
    Hq: int
    Hkv: int
    K: int
    dtype: str
    causal: bool
    past: list
    q_lens: list
    alibi: bool = False
    seed: int = 0
    q: torch.Tensor = field(default=None, repr=False)
    k_new: torch.Tensor = field(default=None, repr=False)
    v_new: torch.Tensor = field(default=None, repr=False)
    k_cache: torch.Tensor = field(default=None, repr=False)
    v_cache: torch.Tensor = field(default=None, repr=False)

    @property
    def scale(self) -> float:
        return self.K ** -0.5


def make_chunk(name, past, M, cap, Hq, Hkv, K, dtype, causal, seed, q_lens=None,
               alibi=False) -> Chunk:
    """Cache rows [0, past[b]) and the chunk are N(0,1); cache rows from past[b] on
    are filled with a constant 3.0 (they are overwritten or never read)."""
    B = len(past)
    q_lens = list(q_lens) if q_lens is not None else [M] * B
    c = Chunk(name, B, M, cap, Hq, Hkv, K, dtype, causal, list(past), q_lens, alibi, seed)
    g = generator(seed)
    c.q = randn((B, M, Hq, K), dtype, g)
    c.k_new = randn((B, M, Hkv, K), dtype, g)
    c.v_new = randn((B, M, Hkv, K), dtype, g)
    c.k_cache = torch.full((B, cap, Hkv, K), 3.0, dtype=DTYPES[dtype])
    c.v_cache = torch.full((B, cap, Hkv, K), 3.0, dtype=DTYPES[dtype])
    for b, p in enumerate(past):
        c.k_cache[b, :p] = randn((p, Hkv, K), dtype, g)
        c.v_cache[b, :p] = randn((p, Hkv, K), dtype, g)
    return c


def chunk_prefill() -> Chunk:
    """Chunked prefill: B=8 sequences with U[1024, 8192] cached rows each take a
    512-row chunk; Hq=32, Hkv=8, K=128, bf16, causal; cache capacity 8704 rows."""
    past = lengths(8, 1024, 8192, generator(1008)).tolist()
    return make_chunk("chunk512_b8_past1k-8k_hq32_hkv8_k128_bf16", past, 512, 8704, 32, 8, 128,
                      "bf16", True, seed=1009)
