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


# ---------------------------------------------------------------------------
# Shaped inputs: score ranges that move across key tiles.  Row maxima of the
# plain N(0,1) draws change little from one key tile to the next; these make
# them climb (or fall) by large factors along the key axis, or put scores in
# the hundreds, or place tile-to-tile jumps of chosen size.
# ---------------------------------------------------------------------------
def ramp(n: int, lo: float, hi: float) -> torch.Tensor:
    """n factors going linearly from lo to hi (float32; lo alone when n == 1)."""
    if n <= 1:
        return torch.full((max(n, 0),), float(lo), dtype=torch.float32)
    return torch.linspace(float(lo), float(hi), n, dtype=torch.float32)


def scale_rows(x: torch.Tensor, factors: torch.Tensor, dim: int = 1) -> torch.Tensor:
    """x with slice i along `dim` multiplied by factors[i] (float32 product, cast
    back to x's dtype)."""
    shape = [1] * x.dim()
    shape[dim] = -1
    return (x.to(torch.float32) * factors.view(shape)).to(x.dtype)


def ramp_keys(p: Prefill, lo: float, hi: float) -> Prefill:
    """Keys of every sequence multiplied by factors going from lo to hi along the
    sequence's key positions (per packed segment when the batch is packed)."""
    if p.seq_lens_q is None:
        f = ramp(p.N, lo, hi)
    else:
        lens = p.seq_lens_k if p.seq_lens_k is not None else p.seq_lens_q
        f = torch.cat([ramp(int(n), lo, hi) for n in lens]) if len(lens) else ramp(0, lo, lo)
    p.k = scale_rows(p.k, f, 1)
    p.name += f"_keys{lo:g}to{hi:g}"
    return p


def amplify(p: Prefill, c: float) -> Prefill:
    """q and k multiplied by c (scores grow by c^2)."""
    p.q = (p.q.to(torch.float32) * c).to(p.q.dtype)
    p.k = (p.k.to(torch.float32) * c).to(p.k.dtype)
    p.name += f"_x{c:g}"
    return p


def ramp_chunk_keys(c: Chunk, lo: float, hi: float) -> Chunk:
    """Cached and new keys multiplied by factors from lo to hi along each
    sequence's key positions 0 .. past + q_len - 1 (the new rows continue the
    cached ones)."""
    for b, (past, n) in enumerate(zip(c.past, c.q_lens)):
        f = ramp(past + n, lo, hi)
        if past:
            c.k_cache[b, :past] = scale_rows(c.k_cache[b, :past], f[:past], 0)
        if n:
            c.k_new[b, :n] = scale_rows(c.k_new[b, :n], f[past:], 0)
    c.name += f"_keys{lo:g}to{hi:g}"
    return c


def tile_step_scores(name: str, B: int, N: int, Hq: int, K: int, dtype: str, steps, tile: int,
                     seed: int, bias: str = "none", noise: float = 0.0) -> Prefill:
    """Scores that are constant within each block of `tile` keys and move by the
    given amounts from block to block: q = e_0 (plus `noise` N(0,1) on the other
    components), key j has component 0 equal to the running sum of steps[:j // tile]
    and N(0,1) elsewhere, so row i's score with key j is exactly that sum (times
    the scale) when noise = 0.  Batch b uses the steps rotated by b.  Values are
    exact in fp16/bf16 when the steps are multiples of 1/16 below 64.  M = N, Hkv = Hq."""
    g = generator(seed)
    p = Prefill(name, B, N, N, Hq, Hq, K, dtype, bias, False, seed)
    q = torch.zeros((B, N, Hq, K), dtype=torch.float32)
    q[..., 0] = 1.0
    if noise:
        q[..., 1:] = noise * torch.randn((B, N, Hq, K - 1), generator=g, dtype=torch.float32)
    k = torch.randn((B, N, Hq, K), generator=g, dtype=torch.float32)
    steps = [float(s) for s in steps]
    nblk = -(-N // tile)
    for b in range(B):
        rot = steps[b % len(steps):] + steps[:b % len(steps)]
        level, levels = 0.0, []
        for t in range(nblk):
            levels.append(level)
            level += rot[t % len(rot)]
        col = torch.tensor(levels, dtype=torch.float32).repeat_interleave(tile)[:N]
        k[b, :, :, 0] = col.view(N, 1)
    p.q = q.to(DTYPES[dtype])
    p.k = k.to(DTYPES[dtype])
    p.v = randn((B, N, Hq, K), dtype, g)
    return p
