"""Parity of the sm_100a prefill kernel (mea_fwd, through the C ABI) with the
fp64 oracle on the same seeded inputs.  Small cases compare every element;
the full-size workloads compare sampled rows the oracle computes one by one."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import BIAS_CODE, Guarded, assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def mea():
    import memory_efficient_exact_mea_b200 as m

    return m


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _run_gpu(mea, p: synth.Prefill):
    """One mea_fwd with out and lse between guard bands (checked untouched)."""
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    kw = {}
    if p.bias.startswith("blockdiag"):
        kw = dict(seqstart_q=p.seqstart_q.to(DEV), seqstart_k=p.seqstart_k.to(DEV))
    go = Guarded((p.B, p.M, p.Hq, p.K), q.dtype, DEV, fill=float("nan"))
    gl = Guarded((p.B, p.Hq, p.M), torch.float32, DEV, fill=float("nan"))
    out, lse = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=p.alibi, out=go.t,
                           lse=gl.t, **kw)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    go.check(p.name + " out")
    gl.check(p.name + " lse")
    return out, lse


def _check_full(mea, orc, p: synth.Prefill, what=None):
    out, lse = _run_gpu(mea, p)
    ref_out, ref_lse = orc.attention(p.q, p.k, p.v, bias=BIAS_CODE[p.bias], scale=p.scale,
                                     alibi=p.alibi, seqstart_q=p.seqstart_q,
                                     seqstart_k=p.seqstart_k)
    what = what or p.name
    assert_out_close(out, ref_out, what)
    assert_lse_close(lse, ref_lse, what)


# --------------------------------------------------------------------------
# Small cases: every element.  Sizes span several 128-row / 128-key tiles and
# ragged tails.
# --------------------------------------------------------------------------
def test_causal_small_workload(mea, orc):
    """B=2, M=N=256, H=8, K=64, fp16, causal: the tutorial's causal example."""
    _check_full(mea, orc, synth.causal_small())


@pytest.mark.parametrize("M", [128, 300, 512])
@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16"), (64, "bf16"), (128, "f16")])
def test_noncausal(mea, orc, M, K, dtype):
    p = synth.make_prefill(f"noncausal_m{M}_k{K}_{dtype}", 2, M, M, 4, 4, K, dtype, "none",
                           seed=10 + M + K)
    _check_full(mea, orc, p)


@pytest.mark.parametrize("M,N", [(200, 333), (333, 200), (1, 700), (129, 129), (640, 1)])
@pytest.mark.parametrize("bias", ["none", "causal"])
def test_rectangular(mea, orc, M, N, bias):
    """M != N: causal is aligned bottom-right (query i sees keys j <= i + N - M)."""
    p = synth.make_prefill(f"rect_{M}x{N}_{bias}", 2, M, N, 4, 2, 128, "bf16", bias,
                           seed=20 + M * 7 + N)
    _check_full(mea, orc, p)


@pytest.mark.parametrize("alibi", [False, True])
@pytest.mark.parametrize("bias", ["none", "causal"])
def test_gqa_alibi_small(mea, orc, alibi, bias):
    p = synth.make_prefill(f"gqa_{bias}_alibi{alibi}", 2, 384, 384, 8, 2, 128, "bf16", bias,
                           alibi=alibi, seed=31)
    _check_full(mea, orc, p)


@pytest.mark.parametrize("K,dtype", [(64, "f16"), (128, "bf16")])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("alibi", [False, True])
def test_varlen(mea, orc, K, dtype, causal, alibi):
    lens = [1, 64, 127, 128, 129, 300, 513, 0, 257]
    p = synth.make_varlen(f"varlen_c{causal}_a{alibi}", lens, 4, 2, K, dtype, causal,
                          seed=40 + K, alibi=alibi)
    _check_full(mea, orc, p)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_different_q_k_lengths(mea, orc, causal):
    """Chunked prefill against a longer key range per sequence."""
    lens_q = [5, 130, 64, 300]
    lens_k = [5, 400, 64, 1000]
    p = synth.make_varlen("varlen_qk", lens_q, 4, 4, 128, "bf16", causal, seed=50,
                          lens_k=lens_k)
    _check_full(mea, orc, p)


def test_strided_layouts(mea, orc):
    """q/k/v as views with non-packed strides ([B, H, S, K] storage permuted)."""
    p = synth.make_prefill("strided", 2, 200, 260, 4, 4, 64, "f16", "causal", seed=60)
    q = p.q.permute(0, 2, 1, 3).contiguous().to(DEV).permute(0, 2, 1, 3)
    k = p.k.permute(0, 2, 1, 3).contiguous().to(DEV).permute(0, 2, 1, 3)
    v = p.v.permute(0, 2, 1, 3).contiguous().to(DEV).permute(0, 2, 1, 3)
    out = torch.empty(2, 4, 200, 64, dtype=torch.float16, device=DEV).permute(0, 2, 1, 3)
    out, lse = mea.mea_fwd(q, k, v, bias="causal", scale=p.scale, out=out)
    torch.cuda.synchronize()
    ref_out, ref_lse = orc.attention(p.q, p.k, p.v, bias=1, scale=p.scale)
    assert_out_close(out, ref_out, "strided")
    assert_lse_close(lse, ref_lse, "strided")


def test_no_keys(mea):
    """N = 0: every row sees no key: out = 0, lse = -inf."""
    q = torch.randn(1, 5, 2, 64, device=DEV, dtype=torch.float16)
    k = torch.empty(1, 0, 2, 64, device=DEV, dtype=torch.float16)
    out, lse = mea.mea_fwd(q, k, k)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    assert torch.all(torch.isneginf(lse))


def test_many_units_per_cta(mea, orc):
    """More 256-row query blocks than SMs, ragged rows and keys: CTAs that run
    several blocks in turn (K=64 fp16 non-causal), every element checked."""
    p = synth.make_prefill("units_b3_h24_m600_n520", 3, 600, 520, 24, 24, 64, "f16", "none", seed=72)
    _check_full(mea, orc, p)


def test_causal_more_queries_than_keys(mea, orc):
    """Causal with M > N: the first M - N rows see no key (out 0, lse -inf)."""
    p = synth.make_prefill("m_gt_n", 1, 300, 100, 2, 2, 64, "f16", "causal", seed=70)
    _check_full(mea, orc, p)


def test_scale_zero_is_mean(mea):
    """Closed form on the GPU path: scale 0 -> out = column mean of v."""
    v = torch.randn(1, 333, 2, 64, device=DEV, dtype=torch.bfloat16)
    q = torch.randn(1, 7, 2, 64, device=DEV, dtype=torch.bfloat16)
    out, lse = mea.mea_fwd(q, v, v, scale=0.0)
    ref = v.double().mean(1, keepdim=True).expand(1, 7, 2, 64)
    assert_out_close(out, ref.cpu(), "scale0")
    assert torch.allclose(lse.double().cpu(), torch.full((1, 2, 7), np.log(333.0),
                                                         dtype=torch.float64), atol=1e-3)


@pytest.mark.parametrize("K,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_scale_zero_causal_is_running_mean(mea, K, dtype):
    """Closed form under a causal mask (diagonal tiles masked): scale 0 -> row i
    is the mean of v_0 .. v_i and lse_i = ln(i + 1)."""
    g = torch.Generator().manual_seed(71)
    M = 300
    v = torch.randn(2, M, 2, K, generator=g).to(dtype)
    q = torch.randn(2, M, 2, K, generator=g).to(dtype)
    out, lse = mea.mea_fwd(q.to(DEV), v.to(DEV), v.to(DEV), bias="causal", scale=0.0)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    cnt = torch.arange(1, M + 1, dtype=torch.float64)
    ref = v.double().cumsum(1) / cnt.view(1, M, 1, 1)
    assert_out_close(out, ref, "scale0_causal")
    assert torch.allclose(lse.double().cpu(), torch.log(cnt).expand(2, 2, M), atol=1e-3)


def test_repeatable(mea):
    """Two launches on the same input give bit-identical results."""
    p = synth.make_prefill("rep", 2, 300, 300, 4, 2, 128, "bf16", "causal", seed=80)
    a = _run_gpu(mea, p)
    b = _run_gpu(mea, p)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# --------------------------------------------------------------------------
# Full-size workloads: sampled rows, computed by the oracle one by one.
# --------------------------------------------------------------------------
def _sample_rows(rng, B, M, Hq, n=192, edges=()):
    rows = [(int(rng.integers(B)), int(rng.integers(M)), int(rng.integers(Hq))) for _ in range(n)]
    for i in edges:
        if 0 <= i < M:
            rows.append((int(rng.integers(B)), i, int(rng.integers(Hq))))
    return np.array(rows, dtype=np.int64)


def _check_sampled(mea, orc, p: synth.Prefill, rows):
    out, lse = _run_gpu(mea, p)
    ref_o, ref_l = orc.attention_rows(p.q, p.k, p.v, rows, bias=BIAS_CODE[p.bias], scale=p.scale,
                                      alibi=p.alibi, seqstart_q=p.seqstart_q,
                                      seqstart_k=p.seqstart_k)
    b, i, h = rows[:, 0], rows[:, 1], rows[:, 2]
    g_out = out.cpu()[b, i, h]
    g_lse = lse.cpu()[b, h, i]
    assert_out_close(g_out, ref_o, p.name)
    assert_lse_close(g_lse, ref_l, p.name)


@pytest.mark.parametrize("M", synth.SWEEP_M)
def test_sweep_full_size_sampled(mea, orc, M):
    p = synth.noncausal_sweep(M)
    rows = _sample_rows(np.random.default_rng(M), p.B, p.M, p.Hq,
                        edges=(0, 127, 128, 255, 256, M - 1))
    _check_sampled(mea, orc, p, rows)


def test_varlen_full_size_sampled(mea, orc):
    p = synth.varlen_causal()
    st = p.seqstart_q.numpy()
    rng = np.random.default_rng(3)
    edges = sorted({int(x) for s in range(len(st) - 1) for x in (st[s], st[s + 1] - 1)})
    rows = _sample_rows(rng, 1, p.M, p.Hq, n=256, edges=edges)
    _check_sampled(mea, orc, p, rows)


def test_gqa_alibi_full_size_sampled(mea, orc):
    p = synth.gqa_alibi_causal()
    rows = _sample_rows(np.random.default_rng(4), p.B, p.M, p.Hq, n=256,
                        edges=(0, 1, 127, 128, 255, 256, 2048, 4095))
    _check_sampled(mea, orc, p, rows)


@pytest.mark.parametrize("K,dtype,bias", [(64, "f16", "none"), (64, "f16", "causal"),
                                          (128, "bf16", "causal")])
def test_repeatable_each_layout(mea, K, dtype, bias):
    """Both TMEM layouts give bit-identical results over repeated launches."""
    p = synth.make_prefill("rep_layout", 2, 700, 650, 4, 2, K, dtype, bias, seed=81)
    first = _run_gpu(mea, p)
    for _ in range(5):
        again = _run_gpu(mea, p)
        assert torch.equal(again[0], first[0]) and torch.equal(again[1], first[1])


@pytest.mark.parametrize("expanded", [False, True])
def test_grouped_5d_layout(mea, orc, expanded):
    """The 5-D grouped-query layout of the xFormers tutorial ("Dimotrazione di
    Gruppo Query Attention (GQA)"): q [B,M,G,H,K] with k, v [B,N,G,1,K] (or expanded
    along H with stride 0).  Query head (g, r) must attend with key/value head g:
    compared with the oracle on the same problem with the key/value heads
    repeated explicitly (every query head its own copy)."""
    B, M, N, G, H, K = 2, 300, 260, 2, 4, 128
    g = synth.generator(90)
    q5 = synth.randn((B, M, G, H, K), "bf16", g)
    k5 = synth.randn((B, N, G, 1, K), "bf16", g)
    v5 = synth.randn((B, N, G, 1, K), "bf16", g)
    kd, vd = k5.to(DEV), v5.to(DEV)
    if expanded:
        kd, vd = kd.expand(B, N, G, H, K), vd.expand(B, N, G, H, K)
    out, lse = mea.mea_fwd(q5.to(DEV), kd, vd, bias="causal", scale=K ** -0.5)
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    assert tuple(out.shape) == (B, M, G, H, K) and tuple(lse.shape) == (B, G * H, M)
    k_rep = k5.expand(B, N, G, H, K).reshape(B, N, G * H, K)
    v_rep = v5.expand(B, N, G, H, K).reshape(B, N, G * H, K)
    ro, rl = orc.attention(q5.reshape(B, M, G * H, K), k_rep, v_rep, bias=1, scale=K ** -0.5)
    assert_out_close(out.reshape(B, M, G * H, K), ro, "5-D grouped")
    assert_lse_close(lse, rl, "5-D grouped")


def test_prepared_call_matches_plain_call(mea):
    """A prepared mea_fwd (arguments marshalled once) gives the plain call's
    results bit for bit, call after call."""
    p = synth.causal_small()
    q, k, v = p.q.to(DEV), p.k.to(DEV), p.v.to(DEV)
    ref = mea.mea_fwd(q, k, v, bias="causal", scale=p.scale)
    call = mea.mea_fwd(q, k, v, bias="causal", scale=p.scale, prepare=True)
    for _ in range(3):
        out, lse = call()
        torch.cuda.synchronize()
        assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])
    assert mea.read_device_status() == 0


@pytest.mark.parametrize("n_seqs", [200, 300])
def test_varlen_many_sequences(mea, orc, n_seqs):
    """Packed causal batches with many sequences (lengths 0 .. 700, a few at the
    maximum): up to 256 sequences the CTAs rank only the units that exist
    (sequences sorted by length), beyond that every (block, head, sequence)
    rank, skipping empty ones.  Every element against the oracle."""
    lens = [int(x) for x in synth.lengths(n_seqs, 0, 700, synth.generator(95 + n_seqs))]
    lens[3] = lens[n_seqs // 2] = 700
    p = synth.make_varlen(f"varlen_{n_seqs}", lens, 4, 2, 64, "f16", True, seed=96)
    _check_full(mea, orc, p)
