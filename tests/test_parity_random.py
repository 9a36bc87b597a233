"""Seeded random configurations of the prefill forward and backward against the
fp64 oracle, element by element: shapes the enumerated tests do not list (odd
head counts and groups, row counts ending anywhere inside a tile, tiny and
rectangular problems, packed batches with empty and one-row sequences, ALiBi
with scales away from 1/sqrt(K)).  Each case is drawn from its own seed, so a
failure names a reproducible configuration.  Method: "FlashAttention (2022)",
"Il trucco della softmax che non ha bisogno di vedere tutto"; packed batches:
"Utilizzare Sequenze di Lunghezza Variabile"."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import BIAS_CODE, Guarded, assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

DEV = "cuda"
N_FWD = 96
N_BWD = 24


@pytest.fixture(scope="module")
def mea():
    import memory_efficient_exact_mea_b200 as m

    return m


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _draw_fwd(case: int):
    """Configuration `case` of the forward sweep (host-side draw, seeded): the
    problem and its softmax scale."""
    rng = np.random.default_rng(9000 + case)
    K = int(rng.choice([64, 128]))
    dtype = str(rng.choice(["f16", "bf16"]))
    Hkv = int(rng.choice([1, 2, 3]))
    Hq = Hkv * int(rng.choice([1, 2, 3, 4]))
    alibi = bool(rng.random() < 0.4)
    causal = bool(rng.random() < 0.5)
    seed = 50000 + case
    if rng.random() < 0.3:  # packed batch
        S = int(rng.integers(1, 6))
        lens = [int(x) for x in rng.integers(0, 420, size=S)]
        lens[int(rng.integers(0, S))] = int(rng.choice([1, 129, 257]))
        p = synth.make_varlen(f"rand{case}_varlen", lens, Hq, Hkv, K, dtype, causal, seed,
                              alibi=alibi)
    else:
        B = int(rng.integers(1, 4))
        M = int(rng.integers(1, 600))
        N = int(rng.integers(1, 600)) if rng.random() < 0.5 else M
        p = synth.make_prefill(f"rand{case}", B, M, N, Hq, Hkv, K, dtype,
                               "causal" if causal else "none", alibi=alibi, seed=seed)
    scale = float(rng.uniform(0.02, 0.4)) if rng.random() < 0.3 else p.scale
    return p, scale


@pytest.mark.parametrize("case", range(N_FWD))
def test_random_forward(mea, orc, case):
    p, scale = _draw_fwd(case)
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    kw = {}
    if p.bias.startswith("blockdiag"):
        kw = dict(seqstart_q=p.seqstart_q.to(DEV), seqstart_k=p.seqstart_k.to(DEV))
    go = Guarded((p.B, p.M, p.Hq, p.K), q.dtype, DEV, fill=float("nan"))
    gl = Guarded((p.B, p.Hq, p.M), torch.float32, DEV, fill=float("nan"))
    out, lse = mea.mea_fwd(q, k, v, bias=p.bias, scale=scale, alibi=p.alibi, out=go.t,
                           lse=gl.t, **kw)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    go.check(p.name + " out")
    gl.check(p.name + " lse")
    ref_out, ref_lse = orc.attention(p.q, p.k, p.v, bias=BIAS_CODE[p.bias], scale=scale,
                                     alibi=p.alibi, seqstart_q=p.seqstart_q,
                                     seqstart_k=p.seqstart_k)
    what = (f"{p.name}: B={p.B} M={p.M} N={p.N} Hq={p.Hq} Hkv={p.Hkv} K={p.K} "
            f"{p.dtype} {p.bias} alibi={p.alibi} scale={scale:.4f}")
    assert_out_close(out, ref_out, what)
    assert_lse_close(lse, ref_lse, what)


def _draw_bwd(case: int) -> synth.Prefill:
    """Configuration `case` of the backward sweep (host-side draw, seeded)."""
    rng = np.random.default_rng(9500 + case)
    K = int(rng.choice([64, 128]))
    dtype = str(rng.choice(["f16", "bf16"]))
    Hkv = int(rng.choice([1, 2]))
    Hq = Hkv * int(rng.choice([1, 2, 3]))
    alibi = bool(rng.random() < 0.4)
    causal = bool(rng.random() < 0.5)
    seed = 60000 + case
    if rng.random() < 0.3:
        lens = [int(x) for x in rng.integers(1, 300, size=int(rng.integers(1, 4)))]
        return synth.make_varlen(f"rand_bwd{case}_varlen", lens, Hq, Hkv, K, dtype, causal, seed,
                                 alibi=alibi)
    B = int(rng.integers(1, 3))
    M = int(rng.integers(1, 330))
    N = int(rng.integers(1, 330)) if rng.random() < 0.5 else M
    return synth.make_prefill(f"rand_bwd{case}", B, M, N, Hq, Hkv, K, dtype,
                              "causal" if causal else "none", alibi=alibi, seed=seed)


@pytest.mark.parametrize("case", range(N_BWD))
def test_random_backward(mea, case):
    from test_parity_bwd import _check

    _check(mea, _draw_bwd(case))
