"""Planted-mistake check for the oracle pins: each mutation swaps one oracle function
for a plausibly wrong variant (on the CPU) and the pins of test_oracle_pins.py must
then fail. A mutation that no pin catches means the pins are too weak.
"""

from __future__ import annotations

import math
from statistics import NormalDist

import numpy as np
import pytest

import oracle
import oracle.wina_oracle as W
from tests import test_oracle_pins as P


def _row_norms(Wm):
    Wm = np.asarray(Wm, dtype=np.float64)
    return np.sqrt((Wm * Wm).sum(axis=1)).astype(np.float32)


def _scores_no_abs(x, c=None):
    x32 = np.asarray(x, dtype=np.float32)
    return x32 if c is None else x32 * np.asarray(c, dtype=np.float32)


def _topk_ties_high(score, k):
    s = np.asarray(score, dtype=np.float32).astype(np.float64)
    n = s.shape[0]
    order = np.lexsort((-np.arange(n), -s))
    return np.sort(order[:k]).astype(np.int32)


def _topk_unsorted(score, k):
    s = np.asarray(score, dtype=np.float32).astype(np.float64)
    n = s.shape[0]
    return np.lexsort((np.arange(n), -s))[:k].astype(np.int32)


def _matvec_rows(Wm, idx, xs):
    # transposed operand: takes row j of W where column j is meant
    Wm = np.asarray(Wm, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size == 0:
        return np.zeros(Wm.shape[1])
    return Wm[idx, :].T @ np.asarray(xs, dtype=np.float64)


def _spark_sample_var(v, s):
    v = np.asarray(v, dtype=np.float64)
    mu = float(v.mean())
    var = float(((v - mu) ** 2).sum() / max(len(v) - 1, 1))
    z = NormalDist().inv_cdf(1.0 - s)
    t = mu + math.sqrt(var) * z
    return dict(mu=mu, var=var, sigma=math.sqrt(var), z=z, t=t, idx=np.nonzero(v > t)[0].astype(np.int32))


def _spark_ge(v, s):
    v = np.asarray(v, dtype=np.float64)
    mu = float(v.mean())
    var = float(((v - mu) ** 2).mean())
    z = NormalDist().inv_cdf(1.0 - s)
    t = mu + math.sqrt(var) * z
    return dict(mu=mu, var=var, sigma=math.sqrt(var), z=z, t=t, idx=np.nonzero(v >= t)[0].astype(np.int32))


def _spark_wrong_tail(v, s):
    v = np.asarray(v, dtype=np.float64)
    mu = float(v.mean())
    var = float(((v - mu) ** 2).mean())
    z = NormalDist().inv_cdf(s)
    t = mu + math.sqrt(var) * z
    return dict(mu=mu, var=var, sigma=math.sqrt(var), z=z, t=t, idx=np.nonzero(v > t)[0].astype(np.int32))


def _silu_minus(g):
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(g))


def _ffn_stat_variant(abs_x=False, up_from_xc=False, h64=False):
    """A copy of the oracle's FFN whose Spark (stat) branch carries one planted mistake:
    gate/up thresholding |x|, the up set taken from x * c_up, or the down gate on the
    float64 h instead of the float32 h held between the projections."""
    real = W.ffn_swiglu

    def ffn(Wg, Wu, Wd, cg, cu, cd, x, kg, ku, kd, mode="topk", s=0.08):
        if mode != "stat":
            return real(Wg, Wu, Wd, cg, cu, cd, x, kg, ku, kd, mode=mode, s=s)
        x = np.asarray(x)
        xv = np.abs(x) if abs_x else x
        ig = W.spark_threshold(xv, s)["idx"]
        iu = W.spark_threshold(np.asarray(x, dtype=np.float32) * np.asarray(cu, dtype=np.float32), s)["idx"] \
            if up_from_xc else ig
        x64 = np.asarray(x, dtype=np.float64)
        g = W.sparse_matvec(Wg, ig, x64[ig])
        u = W.sparse_matvec(Wu, iu, x64[iu])
        h = W.silu(g) * u
        h32 = h.astype(np.float32)
        idn = W.spark_threshold(h if h64 else h32, s)["idx"]
        y = W.sparse_matvec(Wd, idn, h[idn])
        return dict(idx_gate=ig, idx_up=iu, g=g, u=u, h=h, h32=h32, idx_down=idn, y=y)

    return ffn


def _spark_ffn_abs_scores(Wg, Wu, Wd, x, s):
    # thresholds |g| instead of the signed scores
    Wg = np.asarray(Wg, dtype=np.float64)
    x64 = np.asarray(x, dtype=np.float64)
    g = Wg @ x64
    S = W.spark_threshold(np.abs(g).astype(np.float32), s)["idx"]
    u = np.asarray(Wu, dtype=np.float64)[S] @ x64
    h = W.silu(g[S]) * u
    return dict(g=g, g32=g.astype(np.float32), idx=S, u=u, h=h, y=np.asarray(Wd, dtype=np.float64)[:, S] @ h)


def _spark_ffn_swapped_gate(Wg, Wu, Wd, x, s):
    # silu on the up projection instead of the gate
    Wg = np.asarray(Wg, dtype=np.float64)
    x64 = np.asarray(x, dtype=np.float64)
    g = Wg @ x64
    S = W.spark_threshold(g.astype(np.float32), s)["idx"]
    u = np.asarray(Wu, dtype=np.float64)[S] @ x64
    h = W.silu(u) * g[S]
    return dict(g=g, g32=g.astype(np.float32), idx=S, u=u, h=h, y=np.asarray(Wd, dtype=np.float64)[:, S] @ h)


def _svd_transposed(Wm):
    # transposed operand: W V^T instead of W V
    W64 = np.asarray(Wm, dtype=np.float64)
    _, _, vt = np.linalg.svd(W64, full_matrices=False)
    return W64 @ vt, vt.T


MUTATIONS = {
    "col_norms:row-norms": ("col_norms", _row_norms),
    "gate_scores:no-abs": ("gate_scores", _scores_no_abs),
    "select_topk:ties-to-high-index": ("select_topk", _topk_ties_high),
    "select_topk:not-ascending": ("select_topk", _topk_unsorted),
    "sparse_matvec:rows-not-columns": ("sparse_matvec", _matvec_rows),
    "spark:sample-variance": ("spark_threshold", _spark_sample_var),
    "spark:non-strict": ("spark_threshold", _spark_ge),
    "spark:wrong-tail": ("spark_threshold", _spark_wrong_tail),
    "silu:sign": ("silu", _silu_minus),
    "svd_transform:transposed-V": ("svd_transform", _svd_transposed),
    "ffn_swiglu:stat-gate-on-abs-x": ("ffn_swiglu", _ffn_stat_variant(abs_x=True)),
    "ffn_swiglu:stat-up-set-from-x-times-c": ("ffn_swiglu", _ffn_stat_variant(up_from_xc=True)),
    "ffn_swiglu:stat-down-gate-on-float64-h": ("ffn_swiglu", _ffn_stat_variant(h64=True)),
    "spark_ffn:abs-scores": ("spark_ffn", _spark_ffn_abs_scores),
    "spark_ffn:silu-on-up": ("spark_ffn", _spark_ffn_swapped_gate),
}

PINS = [
    P.test_golden_wina_example,
    P.test_golden_spark_examples,
    P.test_col_norms_closed_forms,
    lambda: P.test_select_topk_bruteforce(0),
    P.test_select_ties_lower_index_and_extremes,
    P.test_sparse_matvec_uses_columns_not_rows,
    P.test_silu_closed_forms,
    P.test_ffn_identity_weights_hand_computed,
    P.test_golden_spark_ffn_example,
    P.test_golden_spark_ffn_lookup,
    P.test_gate_scores_single_fp32_multiply,
    lambda: P.test_spark_keep_fraction_gaussian(2304, 2e-3, 0.03),
    P.test_svd_transform_orthogonal_columns_and_norms,
    P.test_svd_transform_keeps_the_output,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(W, attr, bad)
    monkeypatch.setattr(oracle, attr, bad)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except KeyboardInterrupt:
            raise
        except BaseException:  # AssertionError, pytest's Failed, IndexError, ...
            caught += 1
    assert caught > 0, f"no pin caught mutation {name}"


def test_unmutated_oracle_passes_all_pins():
    for pin in PINS:
        pin()
