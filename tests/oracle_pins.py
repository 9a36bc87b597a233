"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with a closed form, an invariant or an independent brute
force.  ``test_oracle_pins.py`` runs them on the real oracle and
``test_oracle_mutants.py`` checks that every planted mistake fails at least one.

Passages (page title, section):
  [cache]   "Transformer : comprendre l'entrainement et l'inference", "Un cache KV simple"
            (scale 1/sqrt(d), tril(diagonal=past_len) mask, -inf fill, softmax, @ v)
  [decode]  same page, "Pre-remplissage et decodage"; and
            "Transformerを実装して少し理解した気になる会(その4)", "KV Cache"
            (decode = the last query row against every cached key)
  [xf]      "Come costruire Transformer efficienti in memoria con xFormers ...":
            causal lower-triangular mask, block-diagonal packed sequences, GQA, ALiBi
  [flash]   "FlashAttention (2022)", "Il trucco della softmax ...": softmax weights
            of a row sum to one; the result is exact.
  [sparse]  "FlashAttention (2022)", "Cosa mostravano i numeri": the block-sparse
            variant leaves out whole blocks of the score matrix; exact otherwise.
  [chunk]   "Transformer : comprendre ...", "Pre-remplissage et decodage" and "Un cache
            KV simple": new keys/values are concatenated after the cached ones and the
            new queries attend under tril(diagonal=past_len).
"""
from __future__ import annotations

import math

import numpy as np

from oracle import BIAS_BLOCKDIAG, BIAS_BLOCKDIAG_CAUSAL, BIAS_CAUSAL, BIAS_NONE

TOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol=TOL, what=""):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        err = np.where(both_inf, 0.0, np.abs(a - b))
    bad = ~(err <= tol * (1.0 + np.abs(np.where(both_inf, 0.0, b))))
    assert not bad.any(), f"{what}: max err {np.nanmax(err)}"


def _offsets(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


# ---------------------------------------------------------------------------
# [flash] weights of a row sum to one: v == 1 gives out == 1 for every row that
# sees at least one key, under every bias kind, GQA and ALiBi.
# ---------------------------------------------------------------------------
def pin_weights_sum_to_one(orc):
    r = _rng(1)
    B, M, N, Hq, Hkv, D = 2, 7, 9, 4, 2, 8
    q, k = r.standard_normal((B, M, Hq, D)), r.standard_normal((B, N, Hkv, D))
    v = np.ones((B, N, Hkv, D))
    for bias in (BIAS_NONE, BIAS_CAUSAL):
        for alibi in (False, True):
            out, lse = orc.attention(q, k, v, bias=bias, alibi=alibi)
            _close(out, np.ones_like(out), what=f"sum-to-one bias={bias} alibi={alibi}")
            assert np.isfinite(lse).all()
    lens_q, lens_k = [3, 1, 5], [4, 2, 6]
    sq, sk = _offsets(lens_q), _offsets(lens_k)
    q1 = r.standard_normal((1, sum(lens_q), Hq, D))
    k1, v1 = r.standard_normal((1, sum(lens_k), Hkv, D)), np.ones((1, sum(lens_k), Hkv, D))
    for bias in (BIAS_BLOCKDIAG, BIAS_BLOCKDIAG_CAUSAL):
        out, _ = orc.attention(q1, k1, v1, bias=bias, seqstart_q=sq, seqstart_k=sk, alibi=True)
        _close(out, np.ones_like(out), what=f"sum-to-one varlen bias={bias}")


# ---------------------------------------------------------------------------
# [cache] causal, M == N: row 0 sees only key 0, so out_0 = v_0 and
# lse_0 = scale <q_0, k_0>.
# ---------------------------------------------------------------------------
def pin_causal_row0_is_v0(orc):
    r = _rng(2)
    B, M, H, D = 2, 6, 3, 8
    q, k, v = (r.standard_normal((B, M, H, D)) for _ in range(3))
    scale = 0.37
    out, lse = orc.attention(q, k, v, bias=BIAS_CAUSAL, scale=scale)
    _close(out[:, 0], v[:, 0], what="causal row 0 == v0")
    _close(lse[:, :, 0], scale * np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]), what="lse row 0")


# ---------------------------------------------------------------------------
# scale = 0 makes every visible score equal, so the output is the plain mean of
# the visible values and lse = ln(#visible).  This pins the mask (which keys
# are visible, bottom-right alignment for M != N, [cache]) and the value rows.
# ---------------------------------------------------------------------------
def pin_scale_zero_means(orc):
    r = _rng(3)
    D, H = 4, 2
    for (M, N) in ((5, 5), (3, 7), (7, 4)):
        q = r.standard_normal((1, M, H, D))
        k, v = r.standard_normal((1, N, H, D)), r.standard_normal((1, N, H, D))
        out, lse = orc.attention(q, k, v, bias=BIAS_NONE, scale=0.0)
        _close(out[0], np.broadcast_to(v[0].mean(0), (M, H, D)), what="mean all")
        _close(lse, np.full((1, H, M), math.log(N)), what="ln N")
        out, lse = orc.attention(q, k, v, bias=BIAS_CAUSAL, scale=0.0)
        for i in range(M):
            n_vis = i + (N - M) + 1  # keys 0 .. i + N - M
            if n_vis <= 0:
                _close(out[0, i], np.zeros((H, D)), what="no key -> 0")
                assert np.all(np.isneginf(lse[0, :, i])), "no key -> lse -inf"
            else:
                _close(out[0, i], v[0, :n_vis].mean(0), what=f"causal mean M={M} N={N} i={i}")
                _close(lse[0, :, i], np.full(H, math.log(n_vis)), what="causal ln count")
    # packed sequences: means over each row's own sequence
    lens_q, lens_k = [2, 4, 3], [3, 4, 1]
    sq, sk = _offsets(lens_q), _offsets(lens_k)
    q = r.standard_normal((1, 9, H, D))
    k, v = r.standard_normal((1, 8, H, D)), r.standard_normal((1, 8, H, D))
    out, lse = orc.attention(q, k, v, bias=BIAS_BLOCKDIAG, scale=0.0, seqstart_q=sq, seqstart_k=sk)
    outc, lsec = orc.attention(q, k, v, bias=BIAS_BLOCKDIAG_CAUSAL, scale=0.0, seqstart_q=sq,
                               seqstart_k=sk)
    for s in range(3):
        vs = v[0, sk[s]:sk[s + 1]]
        m_s, n_s = lens_q[s], lens_k[s]
        for il in range(m_s):
            i = sq[s] + il
            _close(out[0, i], vs.mean(0), what="blockdiag mean")
            _close(lse[0, :, i], np.full(H, math.log(n_s)), what="blockdiag ln")
            n_vis = il + (n_s - m_s) + 1
            if n_vis <= 0:
                assert np.all(np.isneginf(lsec[0, :, i]))
                _close(outc[0, i], np.zeros((H, D)))
            else:
                _close(outc[0, i], vs[:n_vis].mean(0), what="blockdiag causal mean")
                _close(lsec[0, :, i], np.full(H, math.log(n_vis)), what="bd causal ln")


# ---------------------------------------------------------------------------
# [xf] ALiBi with scale 0: weights proportional to r^(pos_i - pos_j) with
# r = exp(-slope_h) over the visible keys -- a geometric series.
# ---------------------------------------------------------------------------
def pin_alibi_geometric(orc):
    r = _rng(4)
    M, N, H, D = 6, 6, 4, 3
    q = r.standard_normal((1, M, H, D))
    k, v = r.standard_normal((1, N, H, D)), r.standard_normal((1, N, H, D))
    slopes = np.array([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)])
    out, lse = orc.attention(q, k, v, bias=BIAS_CAUSAL, scale=0.0, alibi=True)
    for h in range(H):
        ratio = math.exp(-slopes[h])
        for i in range(M):
            w = np.array([ratio ** (i - j) for j in range(i + 1)])
            z = (1.0 - ratio ** (i + 1)) / (1.0 - ratio)
            _close(out[0, i, h], (w[:, None] * v[0, :i + 1, h]).sum(0) / z, what="alibi out")
            _close(lse[0, h, i], math.log(z), what="alibi lse")
    # non-causal: distance is |pos_i - pos_j| on both sides of the diagonal
    out, lse = orc.attention(q, k, v, bias=BIAS_NONE, scale=0.0, alibi=True)
    h, i = 0, 2
    ratio = math.exp(-slopes[h])
    w = np.array([ratio ** abs(i - j) for j in range(N)])
    _close(out[0, i, h], (w[:, None] * v[0, :, h]).sum(0) / w.sum(), what="alibi |i-j|")
    _close(lse[0, h, i], math.log(w.sum()), what="alibi |i-j| lse")


def pin_alibi_slopes(orc):
    """Slopes 2^(-8(h+1)/Hq): Hq=8 gives 1/2 .. 1/256; Hq=16 interleaves the half steps."""
    _close(orc.alibi_slopes(8), [2.0 ** -(h + 1) for h in range(8)], what="slopes Hq=8")
    _close(orc.alibi_slopes(16), [2.0 ** (-(h + 1) / 2.0) for h in range(16)], what="Hq=16")
    _close(orc.alibi_slopes(1), [2.0 ** -8], what="Hq=1")


def pin_alibi_zero_slopes_is_no_bias(orc):
    r = _rng(5)
    q, k, v = (r.standard_normal((2, 5, 4, 8)) for _ in range(3))
    for bias in (BIAS_NONE, BIAS_CAUSAL):
        a = orc.attention(q, k, v, bias=bias, alibi=np.zeros(4))
        b = orc.attention(q, k, v, bias=bias)
        _close(a[0], b[0], what="alibi 0 out")
        _close(a[1], b[1], what="alibi 0 lse")


# ---------------------------------------------------------------------------
# Hand-worked cases.
# ---------------------------------------------------------------------------
def pin_two_key_hand_case(orc):
    """q = e0, k0 = 0, k1 = ln(3) e0, scale 1: scores (0, ln 3) -> weights (1/4, 3/4)."""
    q = np.zeros((1, 1, 1, 2))
    q[0, 0, 0, 0] = 1.0
    k = np.zeros((1, 2, 1, 2))
    k[0, 1, 0, 0] = math.log(3.0)
    v = np.array([[1.0, 2.0], [5.0, -2.0]]).reshape(1, 2, 1, 2)
    out, lse = orc.attention(q, k, v, bias=BIAS_NONE, scale=1.0)
    _close(out[0, 0, 0], [4.0, -1.0], what="hand out")
    _close(lse[0, 0, 0], math.log(4.0), what="hand lse")
    # causal with M=1, N=2: the single query sits at position 1 and sees both keys
    out, _ = orc.attention(q, k, v, bias=BIAS_CAUSAL, scale=1.0)
    _close(out[0, 0, 0], [4.0, -1.0], what="hand causal bottom-right")


def pin_alibi_hand_case(orc):
    """Hq=2 causal, q.k = 0, row 1: scores (-slope_h, 0); slope_0 = 2^-4, slope_1 = 2^-8."""
    q = np.zeros((1, 2, 2, 2))
    k = np.zeros((1, 2, 2, 2))
    v = np.array([[3.0, 1.0], [-1.0, 2.0]])
    vv = np.stack([v, v], axis=1).reshape(1, 2, 2, 2)
    out, lse = orc.attention(q, k, vv, bias=BIAS_CAUSAL, scale=1.0, alibi=True)
    for h, slope in ((0, 2.0 ** -4), (1, 2.0 ** -8)):
        e = math.exp(-slope)
        _close(out[0, 1, h], (e * v[0] + v[1]) / (1.0 + e), what="alibi hand out")
        _close(lse[0, h, 1], math.log(1.0 + e), what="alibi hand lse")


# ---------------------------------------------------------------------------
# Structural invariants.
# ---------------------------------------------------------------------------
def pin_blockdiag_is_independent_runs(orc):
    """[xf] a packed batch with a block-diagonal mask equals one run per sequence."""
    r = _rng(6)
    Hq, Hkv, D = 4, 2, 8
    lens_q, lens_k = [5, 1, 7, 3], [5, 4, 9, 2]
    sq, sk = _offsets(lens_q), _offsets(lens_k)
    q = r.standard_normal((1, sum(lens_q), Hq, D))
    k, v = r.standard_normal((1, sum(lens_k), Hkv, D)), r.standard_normal((1, sum(lens_k), Hkv, D))
    for packed_bias, single_bias in ((BIAS_BLOCKDIAG, BIAS_NONE),
                                     (BIAS_BLOCKDIAG_CAUSAL, BIAS_CAUSAL)):
        for alibi in (False, True):
            out, lse = orc.attention(q, k, v, bias=packed_bias, seqstart_q=sq, seqstart_k=sk,
                                     alibi=alibi)
            for s in range(len(lens_q)):
                qs = q[:, sq[s]:sq[s + 1]]
                ks, vs = k[:, sk[s]:sk[s + 1]], v[:, sk[s]:sk[s + 1]]
                o1, l1 = orc.attention(qs, ks, vs, bias=single_bias, alibi=alibi)
                _close(out[:, sq[s]:sq[s + 1]], o1, what=f"blockdiag seq {s}")
                _close(lse[:, :, sq[s]:sq[s + 1]], l1, what=f"blockdiag lse seq {s}")


def pin_gqa_is_repeated_kv(orc):
    """[xf] query head h reads kv head h // (Hq/Hkv): same as repeating each kv head."""
    r = _rng(7)
    B, M, N, Hq, Hkv, D = 2, 5, 6, 8, 2, 4
    q = r.standard_normal((B, M, Hq, D))
    k, v = r.standard_normal((B, N, Hkv, D)), r.standard_normal((B, N, Hkv, D))
    G = Hq // Hkv
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    for bias in (BIAS_NONE, BIAS_CAUSAL):
        a = orc.attention(q, k, v, bias=bias, alibi=True)
        b = orc.attention(q, kr, vr, bias=bias, alibi=True)
        _close(a[0], b[0], what="gqa out")
        _close(a[1], b[1], what="gqa lse")


def pin_decode_is_last_row(orc):
    """[decode] one decode step equals the last row of a causal prefill over the
    same keys, whose last query is the decode query."""
    r = _rng(8)
    Hq, Hkv, D = 4, 2, 8
    lens = [1, 5, 3, 8]
    st = _offsets(lens)
    T = int(st[-1])
    qd = r.standard_normal((len(lens), Hq, D))
    kc, vc = r.standard_normal((T, Hkv, D)), r.standard_normal((T, Hkv, D))
    for alibi in (False, True):
        out, lse = orc.decode(qd, kc, vc, st, scale=0.3, alibi=alibi)
        for b, n in enumerate(lens):
            qp = r.standard_normal((1, n, Hq, D))
            qp[0, n - 1] = qd[b]
            ks, vs = kc[None, st[b]:st[b + 1]], vc[None, st[b]:st[b + 1]]
            o, l = orc.attention(qp, ks, vs, bias=BIAS_CAUSAL, scale=0.3, alibi=alibi)
            _close(out[b], o[0, n - 1], what=f"decode out b={b}")
            _close(lse[b], l[0, :, n - 1], what=f"decode lse b={b}")
    # an empty cache sees no key
    out, lse = orc.decode(qd[:1], kc[:0], vc[:0], np.array([0, 0], dtype=np.int32))
    _close(out, np.zeros_like(out))
    assert np.isneginf(lse).all()


def pin_key_shift_invariance(orc):
    """Adding one vector u to every key shifts each score of row i by
    scale <q_i, u>: out is unchanged and lse moves by that amount."""
    r = _rng(9)
    q, k, v = (r.standard_normal((1, 5, 2, 4)) for _ in range(3))
    u = r.standard_normal(4)
    for bias in (BIAS_NONE, BIAS_CAUSAL):
        a = orc.attention(q, k, v, bias=bias, scale=0.5)
        b = orc.attention(q, k + u, v, bias=bias, scale=0.5)
        _close(a[0], b[0], tol=1e-10, what="shift out")
        _close(b[1] - a[1], 0.5 * np.einsum("bmhd,d->bhm", q, u), tol=1e-10, what="shift lse")


def pin_rows_match_full(orc):
    """The sampled-row entry point returns the same rows as the full one."""
    r = _rng(10)
    q = r.standard_normal((2, 6, 4, 8))
    k, v = r.standard_normal((2, 7, 2, 8)), r.standard_normal((2, 7, 2, 8))
    rows = np.array([[0, 0, 0], [1, 5, 3], [0, 3, 2], [1, 1, 1]])
    for bias in (BIAS_NONE, BIAS_CAUSAL):
        out, lse = orc.attention(q, k, v, bias=bias, alibi=True)
        o, l = orc.attention_rows(q, k, v, rows, bias=bias, alibi=True)
        _close(o, out[rows[:, 0], rows[:, 1], rows[:, 2]], what="rows out")
        _close(l, lse[rows[:, 0], rows[:, 2], rows[:, 1]], what="rows lse")


# ---------------------------------------------------------------------------
# Brute force: an independent full-matrix formulation with an explicit boolean
# mask (the form of the "Un cache KV simple" listing), on tiny sizes.
# ---------------------------------------------------------------------------
def brute_force(q, k, v, causal, seq_q=None, seq_k=None, slopes=None, scale=None):
    B, M, Hq, D = q.shape
    N, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    G = Hq // Hkv
    if seq_q is None:
        seq_q, seq_k = [M], [N]
    qid = np.repeat(np.arange(len(seq_q)), seq_q)
    kid = np.repeat(np.arange(len(seq_k)), seq_k)
    qpos = np.concatenate([np.arange(m) + (n - m) for m, n in zip(seq_q, seq_k)])
    kpos = np.concatenate([np.arange(n) for n in seq_k])
    allowed = qid[:, None] == kid[None, :]
    if causal:
        allowed &= kpos[None, :] <= qpos[:, None]
    out = np.zeros((B, M, Hq, D))
    lse = np.full((B, Hq, M), -np.inf)
    for b in range(B):
        for h in range(Hq):
            S = scale * (q[b, :, h] @ k[b, :, h // G].T)
            if slopes is not None:
                S = S - slopes[h] * np.abs(qpos[:, None] - kpos[None, :])
            S = np.where(allowed, S, -np.inf)
            for i in range(M):
                if not allowed[i].any():
                    continue
                m = S[i].max()
                e = np.exp(S[i] - m)
                out[b, i, h] = (e / e.sum()) @ v[b, :, h // G]
                lse[b, h, i] = m + math.log(e.sum())
    return out, lse


def pin_brute_force(orc):
    r = _rng(11)
    for (B, M, N, Hq, Hkv, D) in ((2, 5, 5, 4, 2, 8), (1, 3, 8, 2, 1, 4), (2, 8, 3, 3, 3, 5)):
        q = r.standard_normal((B, M, Hq, D))
        k, v = r.standard_normal((B, N, Hkv, D)), r.standard_normal((B, N, Hkv, D))
        slopes = orc.alibi_slopes(Hq)
        for causal in (False, True):
            for sl in (None, slopes):
                o, l = orc.attention(q, k, v, bias=BIAS_CAUSAL if causal else BIAS_NONE,
                                     alibi=sl if sl is not None else None)
                ob, lb = brute_force(q, k, v, causal, slopes=sl)
                _close(o, ob, tol=1e-10, what="brute out")
                _close(l, lb, tol=1e-10, what="brute lse")
    lens_q, lens_k = [3, 2, 6], [4, 2, 5]
    q = r.standard_normal((1, 11, 4, 8))
    k, v = r.standard_normal((1, 11, 2, 8)), r.standard_normal((1, 11, 2, 8))
    for causal in (False, True):
        o, l = orc.attention(q, k, v, bias=BIAS_BLOCKDIAG_CAUSAL if causal else BIAS_BLOCKDIAG,
                             seqstart_q=_offsets(lens_q), seqstart_k=_offsets(lens_k), alibi=True)
        ob, lb = brute_force(q, k, v, causal, lens_q, lens_k, slopes=orc.alibi_slopes(4))
        _close(o, ob, tol=1e-10, what="brute varlen out")
        _close(l, lb, tol=1e-10, what="brute varlen lse")


# ---------------------------------------------------------------------------
# Backward pass: gradients of L = sum(out * dO) with respect to q, k, v.
# ---------------------------------------------------------------------------
def _fd_grads(orc, q, k, v, do, eps=1e-6, **kw):
    """Central finite differences of L through the (separately pinned) forward."""
    def loss(q_, k_, v_):
        return float((orc.attention(q_, k_, v_, **kw)[0] * do).sum())
    grads = []
    for x in (q, k, v):
        g = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if y is x else y for y in (q, k, v)]
            args_m = [xm if y is x else y for y in (q, k, v)]
            g[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        grads.append(g)
    return grads


def pin_bwd_finite_differences(orc):
    """[flash] the recomputed-score backward equals the derivative of the forward."""
    r = _rng(20)
    cases = [
        dict(shape=(1, 3, 4, 2, 1, 3), kw=dict(bias=BIAS_NONE, scale=0.7)),
        dict(shape=(2, 4, 4, 2, 2, 3), kw=dict(bias=BIAS_CAUSAL, scale=0.5, alibi=True)),
        dict(shape=(1, 3, 5, 4, 2, 2), kw=dict(bias=BIAS_CAUSAL, scale=1.1)),
    ]
    for c in cases:
        B, M, N, Hq, Hkv, D = c["shape"]
        q = r.standard_normal((B, M, Hq, D))
        k, v = r.standard_normal((B, N, Hkv, D)), r.standard_normal((B, N, Hkv, D))
        do = r.standard_normal((B, M, Hq, D))
        dq, dk, dv = orc.attention_bwd(q, k, v, do, **c["kw"])
        fq, fk, fv = _fd_grads(orc, q, k, v, do, **c["kw"])
        _close(dq, fq, tol=1e-6, what=f"fd dq {c['kw']}")
        _close(dk, fk, tol=1e-6, what=f"fd dk {c['kw']}")
        _close(dv, fv, tol=1e-6, what=f"fd dv {c['kw']}")
    lens_q, lens_k = [2, 3], [3, 2]
    q = r.standard_normal((1, 5, 2, 2))
    k, v = r.standard_normal((1, 5, 2, 2)), r.standard_normal((1, 5, 2, 2))
    do = r.standard_normal((1, 5, 2, 2))
    for bias in (BIAS_BLOCKDIAG, BIAS_BLOCKDIAG_CAUSAL):
        kw = dict(bias=bias, seqstart_q=_offsets(lens_q), seqstart_k=_offsets(lens_k), scale=0.8)
        got = orc.attention_bwd(q, k, v, do, **kw)
        for g, f, n in zip(got, _fd_grads(orc, q, k, v, do, **kw), "qkv"):
            _close(g, f, tol=1e-6, what=f"fd d{n} varlen bias={bias}")


def pin_bwd_closed_forms(orc):
    """One key: weights are 1, so dq = dk = 0 and dv = sum of dO over the rows and
    query heads reading it.  Constant values: dP_ij = D_i, so dS = 0 (dq = dk = 0)
    and sum_j dv_j = sum_i dO_i."""
    r = _rng(21)
    q = r.standard_normal((2, 4, 4, 3))
    k, v = r.standard_normal((2, 1, 2, 3)), r.standard_normal((2, 1, 2, 3))
    do = r.standard_normal((2, 4, 4, 3))
    dq, dk, dv = orc.attention_bwd(q, k, v, do, scale=0.9)
    _close(dq, np.zeros_like(dq), what="one key dq")
    _close(dk, np.zeros_like(dk), what="one key dk")
    _close(dv[:, 0], do.reshape(2, 4, 2, 2, 3).sum(axis=(1, 3)), what="one key dv")
    k = r.standard_normal((1, 6, 1, 3))
    v = np.broadcast_to(r.standard_normal(3), (1, 6, 1, 3)).copy()
    q, do = r.standard_normal((1, 5, 2, 3)), r.standard_normal((1, 5, 2, 3))
    for bias in (BIAS_NONE, BIAS_CAUSAL):
        dq, dk, dv = orc.attention_bwd(q, k, v, do, bias=bias, alibi=True)
        _close(dq, np.zeros_like(dq), tol=1e-10, what="const v dq")
        _close(dk, np.zeros_like(dk), tol=1e-10, what="const v dk")
        _close(dv.sum(axis=1)[0, 0], do.sum(axis=(0, 1, 2)), tol=1e-10, what="const v sum dv")


def pin_bwd_gqa_and_key_shift(orc):
    """GQA gradients = those of repeated kv heads, with dk/dv summed over each
    group; adding one vector to every key leaves dq and dv unchanged (each row
    of dS sums to zero)."""
    r = _rng(22)
    q, do = r.standard_normal((1, 4, 4, 3)), r.standard_normal((1, 4, 4, 3))
    k, v = r.standard_normal((1, 5, 2, 3)), r.standard_normal((1, 5, 2, 3))
    a = orc.attention_bwd(q, k, v, do, bias=BIAS_CAUSAL, alibi=True)
    b = orc.attention_bwd(q, np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2), do,
                          bias=BIAS_CAUSAL, alibi=True)
    _close(a[0], b[0], tol=1e-10, what="gqa dq")
    _close(a[1], b[1].reshape(1, 5, 2, 2, 3).sum(axis=3), tol=1e-10, what="gqa dk")
    _close(a[2], b[2].reshape(1, 5, 2, 2, 3).sum(axis=3), tol=1e-10, what="gqa dv")
    c = orc.attention_bwd(q, k + r.standard_normal(3), v, do, bias=BIAS_CAUSAL, alibi=True)
    _close(c[0], a[0], tol=1e-9, what="key shift dq")
    _close(c[2], a[2], tol=1e-9, what="key shift dv")


# ---------------------------------------------------------------------------
# [sparse] block-sparse attention = the dense definition with a block mask.
# ---------------------------------------------------------------------------
def pin_block_sparse_reductions(orc):
    """All-ones mask = the dense run; a diagonal block mask = the block-diagonal
    run of the same chunks (rectangular blocks fix which axis is which); under
    causal with square blocks and M = N, = the block-diagonal causal run; a row
    whose blocks are all zero gets out = 0, lse = -inf."""
    r = _rng(30)
    B, M, N, Hq, Hkv, D = 2, 7, 9, 4, 2, 5
    q = r.standard_normal((B, M, Hq, D))
    k, v = r.standard_normal((B, N, Hkv, D)), r.standard_normal((B, N, Hkv, D))
    bm, bn = 2, 4
    ones = np.ones((B, Hq, -(-M // bm), -(-N // bn)), dtype=np.uint8)
    for bias in (BIAS_NONE, BIAS_CAUSAL):
        o, l = orc.attention_block_sparse(q, k, v, ones, bm, bn, bias=bias, alibi=True)
        od, ld = orc.attention(q, k, v, bias=bias, alibi=True)
        _close(o, od, what="all-ones mask out")
        _close(l, ld, what="all-ones mask lse")
    # diagonal: query chunks of 2 rows against key chunks of 3 keys
    q1 = r.standard_normal((1, 6, 2, 4))
    k1, v1 = r.standard_normal((1, 9, 2, 4)), r.standard_normal((1, 9, 2, 4))
    diag = np.broadcast_to(np.eye(3, dtype=np.uint8), (1, 2, 3, 3)).copy()
    o, l = orc.attention_block_sparse(q1, k1, v1, diag, 2, 3, scale=0.7)
    ob, lb = orc.attention(q1, k1, v1, bias=BIAS_BLOCKDIAG, seqstart_q=_offsets([2, 2, 2]),
                           seqstart_k=_offsets([3, 3, 3]), scale=0.7)
    _close(o, ob, what="diagonal mask = blockdiag out")
    _close(l, lb, what="diagonal mask = blockdiag lse")
    q2 = r.standard_normal((1, 9, 2, 4))
    o, l = orc.attention_block_sparse(q2, k1, v1, diag, 3, 3, bias=BIAS_CAUSAL, scale=0.7)
    ob, lb = orc.attention(q2, k1, v1, bias=BIAS_BLOCKDIAG_CAUSAL, seqstart_q=_offsets([3, 3, 3]),
                           seqstart_k=_offsets([3, 3, 3]), scale=0.7)
    _close(o, ob, what="diagonal causal mask out")
    _close(l, lb, what="diagonal causal mask lse")
    holes = ones.copy()
    holes[1, 3, 2, :] = 0  # rows 4, 5 of (b=1, h=3) see nothing
    o, l = orc.attention_block_sparse(q, k, v, holes, bm, bn)
    _close(o[1, 4:6, 3], np.zeros((2, D)), what="empty block row out")
    assert np.all(np.isneginf(l[1, 3, 4:6])), "empty block row lse"
    od, ld = orc.attention(q, k, v)
    _close(o[0], od[0], what="other rows untouched")


def brute_force_block_sparse(q, k, v, mask, bm, bn, causal, scale):
    """Full score matrix with the block mask expanded element by element."""
    B, M, Hq, D = q.shape
    N, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, M, Hq, D))
    lse = np.full((B, Hq, M), -np.inf)
    for b in range(B):
        for h in range(Hq):
            allowed = np.kron(mask[b, h], np.ones((bm, bn)))[:M, :N] > 0
            if causal:
                allowed &= np.arange(N)[None, :] <= np.arange(M)[:, None] + (N - M)
            S = np.where(allowed, scale * (q[b, :, h] @ k[b, :, h // G].T), -np.inf)
            for i in range(M):
                if allowed[i].any():
                    m = S[i].max()
                    e = np.exp(S[i] - m)
                    out[b, i, h] = (e / e.sum()) @ v[b, :, h // G]
                    lse[b, h, i] = m + math.log(e.sum())
    return out, lse


def pin_block_sparse_brute_force(orc):
    """Random per-(batch, head) masks against the expanded-mask brute force; at
    scale 0 every row is the mean of the values it sees and lse = ln(count)."""
    r = _rng(31)
    for (B, M, N, Hq, Hkv, D, bm, bn) in ((2, 7, 10, 4, 2, 3, 3, 4), (1, 9, 5, 2, 1, 4, 2, 2)):
        q = r.standard_normal((B, M, Hq, D))
        k, v = r.standard_normal((B, N, Hkv, D)), r.standard_normal((B, N, Hkv, D))
        mask = (r.random((B, Hq, -(-M // bm), -(-N // bn))) < 0.6).astype(np.uint8)
        for causal in (False, True):
            bias = BIAS_CAUSAL if causal else BIAS_NONE
            o, l = orc.attention_block_sparse(q, k, v, mask, bm, bn, bias=bias, scale=0.9)
            ob, lb = brute_force_block_sparse(q, k, v, mask, bm, bn, causal, 0.9)
            _close(o, ob, tol=1e-10, what="block-sparse brute out")
            _close(l, lb, tol=1e-10, what="block-sparse brute lse")
            rows = np.array([[0, M - 1, Hq - 1], [B - 1, 0, 0], [0, M // 2, 1]])
            orow, lrow = orc.attention_block_sparse(q, k, v, mask, bm, bn, bias=bias, scale=0.9,
                                                    rows=rows)
            _close(orow, o[rows[:, 0], rows[:, 1], rows[:, 2]], what="block-sparse rows out")
            _close(lrow, l[rows[:, 0], rows[:, 2], rows[:, 1]], what="block-sparse rows lse")
            o0, l0 = orc.attention_block_sparse(q, k, v, mask, bm, bn, bias=bias, scale=0.0)
            for b in range(B):
                for h in range(Hq):
                    for i in range(M):
                        keys = [j for j in range(N) if mask[b, h, i // bm, j // bn]
                                and (not causal or j <= i + N - M)]
                        if not keys:
                            assert np.isneginf(l0[b, h, i]) and not o0[b, i, h].any()
                            continue
                        _close(o0[b, i, h], v[b, keys, h // (Hq // Hkv)].mean(axis=0),
                               what="block-sparse scale-0 mean")
                        _close(l0[b, h, i], math.log(len(keys)), what="block-sparse scale-0 lse")


# ---------------------------------------------------------------------------
# [chunk] prefill in chunks against a cache.
# ---------------------------------------------------------------------------
def pin_chunks_equal_full_prefill(orc):
    """Causal prefill of a sequence in two chunks (the second against the cache the
    first one filled) gives the rows of one causal prefill of the whole sequence,
    and leaves the whole sequence's keys/values in the cache (GQA, ALiBi, two
    sequences of different lengths split at different points)."""
    r = _rng(40)
    B, Hq, Hkv, D, cap = 2, 4, 2, 3, 12
    lens, split = [9, 6], [4, 5]
    q_full = r.standard_normal((B, 9, Hq, D))
    k_full, v_full = r.standard_normal((B, 9, Hkv, D)), r.standard_normal((B, 9, Hkv, D))
    kc = np.full((B, cap, Hkv, D), 7.0)
    vc = np.full((B, cap, Hkv, D), -7.0)
    M1, M2 = 5, 5
    q1, k1, v1 = (np.zeros((B, M1) + x.shape[2:]) for x in (q_full, k_full, v_full))
    q2, k2, v2 = (np.zeros((B, M2) + x.shape[2:]) for x in (q_full, k_full, v_full))
    for b in range(B):
        a, n = split[b], lens[b]
        q1[b, :a], k1[b, :a], v1[b, :a] = q_full[b, :a], k_full[b, :a], v_full[b, :a]
        q2[b, :n - a], k2[b, :n - a], v2[b, :n - a] = (q_full[b, a:n], k_full[b, a:n],
                                                       v_full[b, a:n])
    o1, l1, kc, vc = orc.prefill_chunk(q1, k1, v1, kc, vc, [0, 0], q_len=split, alibi=True)
    past = split
    o2, l2, kc, vc = orc.prefill_chunk(q2, k2, v2, kc, vc, past,
                                       q_len=[lens[b] - split[b] for b in range(B)], alibi=True)
    for b in range(B):
        n, a = lens[b], split[b]
        of, lf = orc.attention(q_full[b:b + 1, :n], k_full[b:b + 1, :n], v_full[b:b + 1, :n],
                               bias=BIAS_CAUSAL, alibi=True)
        _close(o1[b, :a], of[0, :a], what="chunk 1 out")
        _close(l1[b, :, :a], lf[0, :, :a], what="chunk 1 lse")
        _close(o2[b, :n - a], of[0, a:n], what="chunk 2 out")
        _close(l2[b, :, :n - a], lf[0, :, a:n], what="chunk 2 lse")
        _close(kc[b, :n], k_full[b, :n], what="cache keys")
        _close(vc[b, :n], v_full[b, :n], what="cache values")
        assert np.all(kc[b, n:] == 7.0) and np.all(vc[b, n:] == -7.0), "rows past the end"
        assert not o2[b, n - a:].any() and np.isnan(l2[b, :, n - a:]).all(), "padding rows"


def pin_chunk_of_one_is_decode(orc):
    """A one-row chunk is a decode step against the cache it extends."""
    r = _rng(41)
    B, Hq, Hkv, D, cap = 3, 4, 2, 5, 10
    past = [0, 4, 9]
    kc, vc = r.standard_normal((B, cap, Hkv, D)), r.standard_normal((B, cap, Hkv, D))
    q, kn, vn = (r.standard_normal((B, 1, H, D)) for H in (Hq, Hkv, Hkv))
    for alibi in (False, True):
        o, l, kc2, vc2 = orc.prefill_chunk(q, kn, vn, kc, vc, past, causal=True, alibi=alibi)
        packed_k = np.concatenate([kc2[b, :past[b] + 1] for b in range(B)])
        packed_v = np.concatenate([vc2[b, :past[b] + 1] for b in range(B)])
        od, ld = orc.decode(q[:, 0], packed_k, packed_v, _offsets([p + 1 for p in past]),
                            alibi=alibi)
        _close(o[:, 0], od, what="one-row chunk = decode out")
        _close(l[:, :, 0], ld, what="one-row chunk = decode lse")


def pin_noncausal_chunk(orc):
    """Without the causal mask a chunk's queries see every cached and new key:
    the plain attention over the concatenation (positions past + i for ALiBi)."""
    r = _rng(42)
    B, M, Hq, Hkv, D, cap = 1, 4, 2, 1, 3, 9
    past = 5
    kc, vc = r.standard_normal((B, cap, Hkv, D)), r.standard_normal((B, cap, Hkv, D))
    q, kn, vn = (r.standard_normal((B, M, H, D)) for H in (Hq, Hkv, Hkv))
    o, l, _, _ = orc.prefill_chunk(q, kn, vn, kc, vc, [past], causal=False, alibi=True)
    k_all = np.concatenate([kc[:, :past], kn], axis=1)
    v_all = np.concatenate([vc[:, :past], vn], axis=1)
    od, ld = orc.attention(q, k_all, v_all, bias=BIAS_NONE, alibi=True)
    _close(o, od, what="non-causal chunk out")
    _close(l, ld, what="non-causal chunk lse")


PINS = [
    pin_weights_sum_to_one,
    pin_causal_row0_is_v0,
    pin_scale_zero_means,
    pin_alibi_geometric,
    pin_alibi_slopes,
    pin_alibi_zero_slopes_is_no_bias,
    pin_two_key_hand_case,
    pin_alibi_hand_case,
    pin_blockdiag_is_independent_runs,
    pin_gqa_is_repeated_kv,
    pin_decode_is_last_row,
    pin_key_shift_invariance,
    pin_rows_match_full,
    pin_brute_force,
    pin_bwd_finite_differences,
    pin_bwd_closed_forms,
    pin_bwd_gqa_and_key_shift,
    pin_block_sparse_reductions,
    pin_block_sparse_brute_force,
    pin_chunks_equal_full_prefill,
    pin_chunk_of_one_is_decode,
    pin_noncausal_chunk,
]
