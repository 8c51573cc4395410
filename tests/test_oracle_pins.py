"""Pins for the CPU oracle: each test checks it against something other than itself
(a hand-worked example, a closed form, brute force, exact integer arithmetic, a
textbook value or a mathematical identity), chosen so that a dropped term, a wrong
sign or index, or a transposed operand in the oracle fails at least one of them.

CPU only (no GPU marker).
"""

from __future__ import annotations

import itertools
import math
import os
from fractions import Fraction
from statistics import NormalDist

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, _, v = line.partition("=")
            out[k.strip()] = [float(t) for t in v.split()]
    return out


# ------------------------------------------------------------------------------------
# storage widening
# ------------------------------------------------------------------------------------


def test_widen_bf16_ieee_values():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0001, 0x7F80, 0x0000, 0x8000], dtype=np.uint16)
    v = O.widen_bf16(bits)
    assert v[0] == 1.0
    assert v[1] == -2.0
    assert v[2] == 1.0 + 2.0 ** -7
    assert v[3] == 2.0 ** -133
    assert math.isinf(v[4]) and v[4] > 0
    assert v[5] == 0.0 and v[6] == 0.0 and math.copysign(1, v[6]) < 0


# ------------------------------------------------------------------------------------
# the hand-worked example (golden fixture)
# ------------------------------------------------------------------------------------


def test_golden_wina_example():
    g = _read_golden("wina_gate_worked_example.txt")
    W = np.array([g["W_row0"], g["W_row1"], g["W_row2"]])
    x = np.array(g["x"], dtype=np.float32)
    c = O.col_norms(W)
    assert c.tolist() == g["c"]
    assert O.gate_scores(x, c).tolist() == g["scores_wina"]
    assert O.gate_scores(x).tolist() == g["scores_teal"]
    for k, key in ((2, "keep_wina_k2"), (3, "keep_wina_k3")):
        idx = O.wina_select(x, c, k)
        assert idx.tolist() == [int(v) for v in g[key]]
    assert O.teal_select(x, 2).tolist() == [int(v) for v in g["keep_teal_k2"]]
    i2 = O.wina_select(x, c, 2)
    i3 = O.wina_select(x, c, 3)
    it = O.teal_select(x, 2)
    assert O.sparse_matvec(W, i2, x[i2]).tolist() == g["y_wina_k2"]
    assert O.sparse_matvec(W, i3, x[i3]).tolist() == g["y_wina_k3"]
    assert O.sparse_matvec(W, it, x[it]).tolist() == g["y_teal_k2"]
    assert O.dense_matvec(W, x).tolist() == g["y_dense"]
    assert O.output_error(W, x, i2) == g["err_wina_k2"][0]
    assert O.output_error(W, x, it) == g["err_teal_k2"][0]


def test_golden_spark_examples():
    g = _read_golden("spark_threshold_worked_example.txt")
    s_a = 1.0 - 0.5 * math.erfc(-1.9 / math.sqrt(2.0))  # 1 - Phi(1.9), via erfc
    r = O.spark_threshold(np.array(g["A_v"]), s_a)
    assert r["mu"] == g["A_mu"][0]
    assert r["var"] == g["A_var"][0]
    assert abs(r["z"] - g["A_z"][0]) < 1e-12
    assert abs(r["t"] - g["A_t"][0]) < 1e-11
    assert r["idx"].tolist() == [int(v) for v in g["A_keep"]]
    r = O.spark_threshold(np.array(g["B_v"]), g["B_s"][0])
    assert r["t"] == g["B_t"][0]
    assert r["idx"].tolist() == [int(v) for v in g["B_keep"]]
    r = O.spark_threshold(np.array(g["C_v"]), g["C_s"][0])
    assert r["sigma"] == 0.0
    assert r["idx"].tolist() == [int(v) for v in g["C_keep"]]


# ------------------------------------------------------------------------------------
# column norms: closed forms and exactly-rounded sums
# ------------------------------------------------------------------------------------


def test_col_norms_closed_forms():
    # non-square on purpose: a row-norm mistake gives a different length and values
    W = np.array([[3.0, 1.0, 0.0, -1.0, 0.0],
                  [4.0, 1.0, 0.0, 1.0, 0.0],
                  [0.0, 1.0, 0.0, -1.0, 6.0],
                  [0.0, 1.0, 0.0, 1.0, 8.0]])
    c = O.col_norms(W)
    assert c.dtype == np.float32
    assert c.tolist() == [5.0, 2.0, 0.0, 2.0, 10.0]
    m = 37
    ones = np.where(np.arange(m)[:, None] % 2 == 0, 1.0, -1.0) * np.ones((m, 3))
    assert np.array_equal(O.col_norms(ones), np.full(3, np.float32(math.sqrt(m))))


def test_col_norms_vs_exact_sum():
    rng = np.random.default_rng(123)
    W = (rng.standard_normal((300, 17)) * rng.lognormal(0, 0.5, 17)).astype(np.float32)
    c = O.col_norms(W)
    for j in range(W.shape[1]):
        exact = Fraction(0)
        for v in W[:, j].astype(np.float64):
            exact += Fraction(float(v)) ** 2
        # sqrt of the exactly rounded fp64 sum, then one rounding to fp32
        want = np.float32(math.sqrt(float(exact)))
        assert c[j] == want, (j, c[j], want)


# ------------------------------------------------------------------------------------
# the gate: scores and top-K against brute force
# ------------------------------------------------------------------------------------


def test_gate_scores_single_fp32_multiply():
    x = np.array([1.5, -2.0, 0.1, -0.0], dtype=np.float32)
    c = np.array([2.0, 3.0, 3.0, 5.0], dtype=np.float32)
    s = O.gate_scores(x, c)
    assert s.dtype == np.float32
    assert s[0] == 3.0 and s[1] == 6.0
    assert s[2] == np.float32(np.float32(0.1) * np.float32(3.0))
    assert s[3] == 0.0 and math.copysign(1, float(s[3])) > 0
    assert O.gate_scores(x).tolist() == [1.5, 2.0, np.float32(0.1), 0.0]


def _brute_topk(score, k):
    """Max-sum K-subset; among equal sums the lexicographically smallest index tuple
    (itertools.combinations enumerates in lexicographic order)."""
    best, best_sum = (), None
    for comb in itertools.combinations(range(len(score)), k):
        s = sum(score[i] for i in comb)
        if best_sum is None or s > best_sum:
            best, best_sum = comb, s
    return list(best)


@pytest.mark.parametrize("seed", range(6))
def test_select_topk_bruteforce(seed):
    rng = np.random.default_rng(seed)
    for n in range(0, 11):
        # integer-valued scores from a tiny alphabet: many ties, exact sums
        score = rng.integers(0, 4, size=n).astype(np.float32)
        for k in range(0, n + 1):
            assert O.select_topk(score, k).tolist() == _brute_topk([int(v) for v in score], k)
        # dyadic continuous scores: exact sums, rare ties
        score = (rng.integers(0, 1 << 12, size=n) / 64.0).astype(np.float32)
        for k in range(0, n + 1):
            assert O.select_topk(score, k).tolist() == _brute_topk([Fraction(float(v)) for v in score], k)


def test_select_ties_lower_index_and_extremes():
    x = np.full(9, 0.5, dtype=np.float32)
    c = np.ones(9, dtype=np.float32)
    assert O.wina_select(x, c, 4).tolist() == [0, 1, 2, 3]
    assert O.wina_select(x, c, 0).tolist() == []
    assert O.wina_select(x, c, 9).tolist() == list(range(9))
    with pytest.raises(ValueError):
        O.select_topk(x, 10)


def test_wina_differs_from_teal_when_norms_differ():
    # |x| favours channel 0, |x c| favours channel 1
    x = np.array([2.0, 1.0], dtype=np.float32)
    c = np.array([1.0, 4.0], dtype=np.float32)
    assert O.wina_select(x, c, 1).tolist() == [1]
    assert O.teal_select(x, 1).tolist() == [0]


# ------------------------------------------------------------------------------------
# the sparse product against exact integer arithmetic
# ------------------------------------------------------------------------------------


def test_sparse_matvec_exact_integers():
    rng = np.random.default_rng(7)
    m, n = 13, 21
    W = rng.integers(-50, 51, size=(m, n))
    x = rng.integers(-9, 10, size=n)
    for k in (0, 1, 5, n):
        idx = np.sort(rng.choice(n, size=k, replace=False))
        want = [sum(int(W[i, j]) * int(x[j]) for j in idx) for i in range(m)]
        got = O.sparse_matvec(W.astype(np.float64), idx, x[idx].astype(np.float64))
        assert got.tolist() == want
    # K = n is the dense product; K = 0 is zero
    full = [sum(int(W[i, j]) * int(x[j]) for j in range(n)) for i in range(m)]
    assert O.dense_matvec(W, x).tolist() == full
    assert O.sparse_matvec(W, np.arange(n), x).tolist() == full
    assert not O.sparse_matvec(W, np.zeros(0, dtype=np.int32), np.zeros(0)).any()


def test_sparse_matvec_uses_columns_not_rows():
    # a transposed operand would pick row j instead of column j
    W = np.array([[1.0, 2.0, 3.0],
                  [4.0, 5.0, 6.0]])
    assert O.sparse_matvec(W, [2], [1.0]).tolist() == [3.0, 6.0]


def test_union_indices():
    assert O.union_indices([[3, 1], [1, 7], []]).tolist() == [1, 3, 7]
    assert O.union_indices([]).tolist() == []


# ------------------------------------------------------------------------------------
# the WINA theorem (section 二) on column-orthogonal W
# ------------------------------------------------------------------------------------


def _col_orthogonal(rng, m, n, d=None):
    q, _ = np.linalg.qr(rng.standard_normal((m, n)))
    if d is None:
        d = rng.lognormal(0.0, 0.5, size=n)
    return q * d[None, :], d


def test_error_identity_column_orthogonal():
    # ||W(x - m.x)||^2 = sum over dropped i of (x_i ||W_i||)^2 when W^T W is diagonal
    rng = np.random.default_rng(11)
    W, d = _col_orthogonal(rng, 40, 24)
    x = rng.laplace(size=24)
    S = np.sort(rng.choice(24, size=10, replace=False))
    dropped = np.setdiff1d(np.arange(24), S)
    want = float(np.sum((x[dropped] * d[dropped]) ** 2))
    assert abs(O.output_error(W, x, S) - want) <= 1e-10 * want


def test_wina_is_error_argmin_bruteforce():
    rng = np.random.default_rng(5)
    for trial in range(20):
        n, m = 8, 12
        W, _ = _col_orthogonal(rng, m, n)
        x = rng.laplace(size=n)
        c = O.col_norms(W)
        for k in range(0, n + 1):
            errs = {comb: O.output_error(W, x, list(comb)) for comb in itertools.combinations(range(n), k)}
            best = min(errs.values())
            wina = tuple(O.wina_select(x.astype(np.float32), c, k).tolist())
            assert errs[wina] <= best * (1 + 1e-9) + 1e-12, (trial, k)


def test_wina_error_le_teal_every_draw():
    # the theorem's claim, checked on every one of 10^4 seeded draws (n = 256)
    rng = np.random.default_rng(2024)
    n, m, k = 256, 320, 96
    draws = 0
    for _ in range(50):
        W, _ = _col_orthogonal(rng, m, n)
        c = O.col_norms(W)
        X = rng.laplace(size=(200, n))
        for x in X:
            ew = O.output_error(W, x, O.wina_select(x.astype(np.float32), c, k))
            et = O.output_error(W, x, O.teal_select(x.astype(np.float32), k))
            assert ew <= et * (1 + 1e-9), (ew, et)
            draws += 1
    assert draws == 10_000


def test_equal_norms_wina_equals_teal():
    # W^T W = I (the theorem's literal hypothesis): all c_i = 1 and the gates coincide
    rng = np.random.default_rng(3)
    n = 64
    ones = np.ones(n, dtype=np.float32)
    for _ in range(50):
        x = rng.laplace(size=n).astype(np.float32)
        for k in (0, 1, 17, 63, 64):
            assert np.array_equal(O.wina_select(x, ones, k), O.teal_select(x, k))


def test_wina_beats_teal_on_average_nonorthogonal():
    # not a theorem on general W: an empirical check on the synthetic weight recipe
    rng = np.random.default_rng(9)
    n, m, k = 256, 512, 128
    W = rng.standard_normal((m, n)) * rng.lognormal(0, 0.5, n)[None, :]
    c = O.col_norms(W)
    ratios = []
    for _ in range(200):
        x = rng.laplace(size=n)
        ew = O.output_error(W, x, O.wina_select(x.astype(np.float32), c, k))
        et = O.output_error(W, x, O.teal_select(x.astype(np.float32), k))
        ratios.append(ew / et)
    assert np.mean(ratios) < 1.0


# ------------------------------------------------------------------------------------
# Spark statistical top-k (section 2.2)
# ------------------------------------------------------------------------------------


def test_normal_quantile_textbook_values():
    nd = NormalDist()
    assert nd.inv_cdf(0.5) == 0.0
    assert abs(nd.inv_cdf(0.975) - 1.959963984540054) < 1e-13
    assert abs(nd.inv_cdf(0.95) - 1.6448536269514722) < 1e-13
    for s in (0.08, 0.01, 0.15, 0.5, 0.9):
        z = O.spark_threshold(np.array([0.0, 1.0]), s)["z"]
        # round trip through the closed form Phi(z) = erfc(-z / sqrt 2) / 2
        assert abs(0.5 * math.erfc(-z / math.sqrt(2.0)) - (1.0 - s)) < 1e-14


@pytest.mark.parametrize("n,mean_tol,band", [(9216, 1e-3, 0.02), (2304, 2e-3, 0.03)])
def test_spark_keep_fraction_gaussian(n, mean_tol, band):
    s = 0.08
    rng = np.random.default_rng(n)
    fracs = []
    for _ in range(1000):
        mu = rng.uniform(-0.1, 0.1)
        sig = rng.uniform(0.5, 2.0)
        v = mu + sig * rng.standard_normal(n)
        fracs.append(len(O.spark_threshold(v, s)["idx"]) / n)
    fracs = np.array(fracs)
    assert abs(fracs.mean() - s) <= mean_tol
    assert fracs.min() >= s - band and fracs.max() <= s + band


def test_spark_scale_and_shift_invariance():
    # the kept set of a*v + b (a > 0) equals that of v: t moves with mu and sigma
    rng = np.random.default_rng(1)
    v = rng.standard_normal(1000)
    base = O.spark_threshold(v, 0.1)["idx"]
    for a, b in ((2.0, 0.0), (0.5, 3.0), (8.0, -1.0)):
        assert np.array_equal(O.spark_threshold(a * v + b, 0.1)["idx"], base)
    # a < 0 mirrors the distribution: the kept set comes from the other tail
    neg = O.spark_threshold(-v, 0.1)["idx"]
    assert set(neg.tolist()).isdisjoint(base.tolist())


def test_spark_nested_with_exact_topk():
    # both sets are upper level sets of one vector, so one contains the other
    rng = np.random.default_rng(4)
    for n in (2304, 9216):
        k = int(math.floor(0.08 * n + 0.5))
        for _ in range(20):
            v = (rng.uniform(-0.1, 0.1) + rng.uniform(0.5, 2) * rng.standard_normal(n)).astype(np.float32)
            S = O.spark_threshold(v, 0.08)["idx"]
            T = O.exact_topk_signed(v, k)
            ov = O.overlap(S, T)
            assert ov["inter"] == min(len(S), k)
            assert ov["jaccard"] == min(len(S), k) / max(len(S), k)


# ------------------------------------------------------------------------------------
# SwiGLU composition
# ------------------------------------------------------------------------------------


def test_silu_closed_forms():
    assert O.silu(0.0) == 0.0
    ln3 = math.log(3.0)
    assert abs(O.silu(ln3) - 0.75 * ln3) < 1e-15  # sigmoid(ln 3) = 3/4
    g = np.linspace(-6, 6, 25)
    assert np.allclose(O.silu(-g), O.silu(g) - g, rtol=0, atol=1e-14)  # sigmoid(-g) = 1 - sigmoid(g)
    assert O.silu(-800.0) == 0.0


def test_ffn_identity_weights_hand_computed():
    # W_gate = W_up = W_down = I (4x4), c = 1, K_gate = K_up = 2, K_down = 1
    x = np.array([1.0, -2.0, 0.5, 3.0], dtype=np.float32)
    eye = np.eye(4)
    one = np.ones(4, dtype=np.float32)
    r = O.ffn_swiglu(eye, eye, eye, one, one, one, x, 2, 2, 1)
    assert r["idx_gate"].tolist() == [1, 3] and r["idx_up"].tolist() == [1, 3]
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))  # noqa: E731
    h1 = (-2.0 * sig(-2.0)) * -2.0  # silu(g) * u with g = u = -2
    h3 = (3.0 * sig(3.0)) * 3.0
    assert np.allclose(r["h"], [0.0, h1, 0.0, h3], rtol=1e-15, atol=0)
    assert r["idx_down"].tolist() == [3]
    assert np.allclose(r["y"], [0.0, 0.0, 0.0, h3], rtol=1e-15, atol=0)
    # no sparsity: y = silu(x) * x elementwise
    r = O.ffn_swiglu(eye, eye, eye, one, one, one, x, 4, 4, 4)
    xd = x.astype(np.float64)
    assert np.allclose(r["y"], (xd / (1 + np.exp(-xd))) * xd, rtol=1e-15, atol=0)


def _zstar_exact(v, i):
    """(v_i - mean) / std of v in exact rational arithmetic, square root to 60 digits."""
    from decimal import Decimal, localcontext

    fv = [Fraction(float(a)) for a in v]
    n = len(fv)
    mu = sum(fv) / n
    var = sum((a - mu) ** 2 for a in fv) / n
    with localcontext() as ctx:
        ctx.prec = 60
        num = Decimal((fv[i] - mu).numerator) / Decimal((fv[i] - mu).denominator)
        return num / (Decimal(var.numerator) / Decimal(var.denominator)).sqrt()


def test_golden_spark_ffn_example():
    # Spark gate on every projection of a SwiGLU FFN with identity weights: gate and up
    # share the set of the signed x, the down gate thresholds the float32 h
    g = _read_golden("spark_ffn_worked_example.txt")
    eye = np.eye(6)
    x = np.array(g["x"], dtype=np.float32)
    assert float(x[4]) == 41.0 + 2.0 ** -18
    cg = np.ones(6, dtype=np.float32)
    cu = np.array(g["c_up"], dtype=np.float32)
    cd = np.ones(6, dtype=np.float32)
    s = g["s"][0]
    # the knife edge, independently of the oracle: the stdlib quantile of 1 - s lies
    # strictly between the exact cut points of the float64 and the float32 h4
    from decimal import Decimal

    z = Decimal(NormalDist().inv_cdf(1.0 - s))
    h64 = [0.0, 0.0, 0.0, 0.0, (41.0 + 2.0 ** -18) ** 2, 2500.0]
    h32 = [float(np.float32(a)) for a in h64]
    assert h32[4] == g["h4_float32"][0] and h64[4] == g["y"][4]
    z32, z64 = _zstar_exact(h32, 4), _zstar_exact(h64, 4)
    assert abs(z32 - Decimal(g["zstar_float32"][0])) < Decimal("1e-15")
    assert abs(z64 - Decimal(g["zstar_float64"][0])) < Decimal("1e-15")
    assert z64 < z < z32
    r = O.ffn_swiglu(eye, eye, eye, cg, cu, cd, x, 0, 0, 0, mode="stat", s=s)
    assert r["idx_gate"].tolist() == [int(v) for v in g["keep_gate"]]
    assert r["idx_up"].tolist() == [int(v) for v in g["keep_up"]]
    assert r["idx_down"].tolist() == [int(v) for v in g["keep_down"]]
    assert r["y"].tolist() == g["y"]


def test_golden_spark_ffn_lookup():
    # Spark FFN as a key-value lookup: dense scores, statistical top-k on them, only the
    # selected neurons' up rows and down columns used
    g = _read_golden("spark_ffn_lookup_worked_example.txt")
    x = np.array(g["x"])
    Wg = np.array([g[f"Wg_row{i}"] for i in range(5)])
    Wu = np.full((5, 3), 9.0)
    Wu[3], Wu[4] = g["Wu_row3"], g["Wu_row4"]
    Wd = np.full((3, 5), 5.0)
    Wd[:, 3], Wd[:, 4] = g["Wd_col3"], g["Wd_col4"]
    s = 0.5 * math.erfc(g["z"][0] / math.sqrt(2.0))  # 1 - Phi(z)
    r = O.spark_ffn(Wg, Wu, Wd, x, s)
    assert r["g"].tolist() == [-2.0, 0.0, 1.0, 4.0, 7.0]
    assert r["idx"].tolist() == [int(v) for v in g["keep"]]
    h3 = 16.0 / (1.0 + math.exp(-4.0))
    h4 = 7.0 / (1.0 + math.exp(-7.0))
    assert np.allclose(r["h"], [h3, h4], rtol=1e-15, atol=0)
    assert np.allclose(r["y"], [h3, h4, 2 * h3 + h4], rtol=1e-15, atol=0)


def test_ffn_gate_and_up_use_their_own_norms():
    # gate and up see the same x but different c: their kept sets must differ
    x = np.array([1.0, 1.0, 1.0, 1.0], dtype=np.float32)
    eye = np.eye(4)
    cg = np.array([4, 3, 2, 1], dtype=np.float32)
    cu = np.array([1, 2, 3, 4], dtype=np.float32)
    r = O.ffn_swiglu(eye, eye, eye, cg, cu, np.ones(4, dtype=np.float32), x, 2, 2, 4)
    assert r["idx_gate"].tolist() == [0, 1]
    assert r["idx_up"].tolist() == [2, 3]
    # gate and up outputs never overlap here, so h = 0 everywhere
    assert not r["h"].any()


# ------------------------------------------------------------------------------------
# the column-orthogonalising transform ([WINA] section 五)
# ------------------------------------------------------------------------------------


def test_svd_transform_orthogonal_columns_and_norms():
    rng = np.random.default_rng(31)
    W = rng.standard_normal((40, 16)) * rng.lognormal(0.0, 0.5, size=16)  # correlated scales
    Wp, V = O.svd_transform(W)
    s = np.linalg.svd(W, compute_uv=False)
    G = Wp.T @ Wp
    off = G - np.diag(np.diag(G))
    assert np.abs(off).max() <= 1e-10 * s[0] ** 2
    assert np.allclose(np.diag(G), s**2, rtol=1e-10)
    assert np.allclose(V.T @ V, np.eye(16), atol=1e-12)  # V is orthogonal
    # the gate's column norms of W' are the singular values (one rounding to float32)
    assert np.allclose(O.col_norms(Wp), s.astype(np.float32), rtol=1e-6)


def test_svd_transform_keeps_the_output():
    rng = np.random.default_rng(32)
    W = rng.standard_normal((30, 12))
    x = rng.laplace(size=12)
    Wp, V = O.svd_transform(W)
    y = O.dense_matvec(W, x)
    assert np.allclose(O.dense_matvec(Wp, V.T @ x), y, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_svd_transform_makes_wina_the_error_minimiser():
    # on a non-orthogonal W the WINA set need not minimise the output error; after the
    # transform (gate on W' and x' = V^T x) it does, for every K (brute force, n = 8)
    rng = np.random.default_rng(33)
    for trial in range(10):
        W = rng.standard_normal((12, 8)) @ rng.standard_normal((8, 8))  # correlated columns
        Wp, V = O.svd_transform(W)
        xp = V.T @ rng.laplace(size=8)
        c = O.col_norms(Wp)
        for k in range(0, 9):
            errs = {comb: O.output_error(Wp, xp, list(comb)) for comb in itertools.combinations(range(8), k)}
            best = min(errs.values())
            wina = tuple(O.wina_select(xp.astype(np.float32), c, k).tolist())
            assert errs[wina] <= best * (1 + 1e-6) + 1e-12, (trial, k)
