"""Pins for the Double Sparsity decode oracle ("大模型DoubleSparse稀疏化技术原理",
sections 离线校准 and 在线前向计算), each against something other than the oracle itself:
a hand-worked example, closed forms, brute force over token subsets, and the special
cases that reduce to plain softmax attention (checked against torch's
scaled_dot_product_attention on the CPU). Planted mistakes in the oracle must fail a pin.
"""

from __future__ import annotations

import itertools
import math
import os

import numpy as np
import pytest

import oracle as O
import oracle.ds_oracle as D

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


def _golden_case():
    g = _read_golden("ds_decode_worked_example.txt")
    K = np.array([g[f"K{t}"] for t in range(5)], dtype=np.float32)
    V = np.array([g["V0"], g["Vother"], g["V2"], g["Vother"], g["Vother"]], dtype=np.float32)
    q = np.array(g["q"], dtype=np.float32)
    C = np.array(g["channels"], dtype=np.int32)
    return g, q, K, V, C


def pin_golden():
    g, q, K, V, C = _golden_case()
    lab = O.ds_label_cache(K, C)
    r = O.ds_decode_head(q, K, V, lab, C, int(g["k"][0]))
    assert np.array_equal(r["scores"], np.array(g["scores"], dtype=np.float32))
    assert np.array_equal(r["idx"], np.array(g["keep"], dtype=np.int32))
    assert np.allclose(r["out"], g["out"], rtol=0, atol=1e-15)


def _sdpa(q, K, V, scale=None):
    torch = pytest.importorskip("torch")
    qt = torch.tensor(q, dtype=torch.float64).view(1, 1, 1, -1)
    Kt = torch.tensor(K, dtype=torch.float64).view(1, 1, K.shape[0], -1)
    Vt = torch.tensor(V, dtype=torch.float64).view(1, 1, V.shape[0], -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o.view(-1).numpy()


def pin_full_attention():
    """Every channel important and k = T: plain softmax attention over all tokens."""
    rng = np.random.default_rng(1)
    for T, dh in ((7, 8), (33, 16), (100, 64)):
        q = rng.standard_normal(dh).astype(np.float32)
        K = rng.standard_normal((T, dh)).astype(np.float32)
        V = rng.standard_normal((T, dh)).astype(np.float32)
        C = np.arange(dh, dtype=np.int32)
        for k in (T, T + 5):
            r = O.ds_decode_head(q, K, V, O.ds_label_cache(K, C), C, k)
            assert np.allclose(r["out"], _sdpa(q, K, V), rtol=1e-12, atol=1e-12)


def pin_selected_subset_attention():
    """Attention over a subset equals softmax attention over that subset alone."""
    rng = np.random.default_rng(2)
    T, dh = 40, 16
    q = rng.standard_normal(dh).astype(np.float32)
    K = rng.standard_normal((T, dh)).astype(np.float32)
    V = rng.standard_normal((T, dh)).astype(np.float32)
    C = np.array([1, 4, 9], dtype=np.int32)
    r = O.ds_decode_head(q, K, V, O.ds_label_cache(K, C), C, 6)
    assert r["idx"].size == 6
    assert np.allclose(r["out"], _sdpa(q, K[r["idx"]], V[r["idx"]]), rtol=1e-12, atol=1e-12)
    # an explicit scale is used as given
    r2 = O.ds_attention(q, K, V, r["idx"], scale=0.3)
    assert np.allclose(r2, _sdpa(q, K[r["idx"]], V[r["idx"]], scale=0.3), rtol=1e-12, atol=1e-12)


def pin_k1_is_argmax_value_row():
    """k = 1: the softmax over one token is 1, so the output is that token's value row,
    the token of largest approximate score (lowest index among equals)."""
    rng = np.random.default_rng(3)
    T, dh, C = 30, 8, np.array([0, 5], dtype=np.int32)
    q = rng.standard_normal(dh).astype(np.float32)
    K = rng.integers(-3, 4, size=(T, dh)).astype(np.float32)  # integer scores: many ties
    V = rng.standard_normal((T, dh)).astype(np.float32)
    r = O.ds_decode_head(q, K, V, O.ds_label_cache(K, C), C, 1)
    s = q[0] * K[:, 0] + q[5] * K[:, 5]
    best = int(np.flatnonzero(s == s.max())[0])
    assert r["idx"].tolist() == [best]
    assert np.array_equal(r["out"], V[best].astype(np.float64))


def pin_selection_brute_force():
    """On tiny T the kept set is the k-subset of largest score sum, ties broken toward the
    lexicographically smallest index set (i.e. lower indices first)."""
    rng = np.random.default_rng(4)
    for _ in range(30):
        T = int(rng.integers(1, 9))
        s = rng.integers(-3, 4, size=T).astype(np.float32)  # ties
        for k in range(0, T + 1):
            best = max(itertools.combinations(range(T), k),
                       key=lambda S: (sum(s[list(S)]), [-i for i in S]))
            assert O.ds_select_tokens(s, k).tolist() == list(best)


def pin_score_order():
    """The approximate score is a float32 sum in channel order with a rounding after
    each add: (1e8 + 1) rounds to 1e8 in float32, so 1e8 + 1 - 1e8 scores 0, where the
    exact sum is 1 and the reverse order gives 1 too."""
    q = np.array([1.0, 1.0, 1.0], dtype=np.float32)
    lab = np.array([[1e8, 1.0, -1e8], [-1e8, 1.0, 1e8], [1.0, 2.0, 3.0]], dtype=np.float32)
    s = O.ds_scores(q, lab, np.array([0, 1, 2]))
    assert s.dtype == np.float32
    assert s.tolist() == [0.0, 0.0, 6.0]
    # products are rounded to float32 before the add
    q2 = np.array([1.0 + 2.0 ** -12], dtype=np.float32)
    lab2 = np.array([[1.0 + 2.0 ** -12]], dtype=np.float32)
    assert O.ds_scores(q2, lab2, np.array([0]))[0] == np.float32((1.0 + 2.0 ** -12) ** 2)


def pin_label_and_calibration():
    """The label cache is the chosen channels of K; K-outlier calibration picks the
    channels of largest mean |K| (ties to the lower channel), ascending."""
    rng = np.random.default_rng(5)
    T, dh = 64, 32
    K = rng.uniform(-1, 1, size=(T, dh)).astype(np.float32)
    big = [3, 17, 30, 8]
    K[:, big] *= 10
    assert O.ds_calibrate_channels(K, 4).tolist() == sorted(big)
    lab = O.ds_label_cache(K, np.array(sorted(big)))
    assert np.array_equal(lab, K[:, sorted(big)])
    # sign does not matter, magnitude does; exact ties go to the lower channel
    K2 = np.zeros((4, 6), dtype=np.float32)
    K2[:, 5] = -2.0
    K2[:, 1] = 2.0
    K2[:, 3] = 1.0
    assert O.ds_calibrate_channels(K2, 2).tolist() == [1, 5]
    assert O.ds_calibrate_channels(K2, 3).tolist() == [1, 3, 5]
    assert O.ds_calibrate_channels(K2, 4).tolist() == [0, 1, 3, 5]


def pin_batch_gqa_layout():
    """The batched call equals the per-head call with query head h reading key/value head
    h // (Hq / Hkv), over each sequence's own length."""
    rng = np.random.default_rng(6)
    B, Hq, Hkv, Tm, dh, r, k = 2, 4, 2, 20, 8, 3, 5
    q = rng.standard_normal((B, Hq, dh)).astype(np.float32)
    K = rng.standard_normal((B, Hkv, Tm, dh)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, Tm, dh)).astype(np.float32)
    C = np.array([[0, 2, 7], [1, 3, 5]], dtype=np.int32)
    lab = np.stack([np.stack([K[b, g][:, C[g]] for g in range(Hkv)]) for b in range(B)])
    seq = [20, 9]
    r = O.ds_decode(q, K, V, lab, C, seq, k)
    for b in range(B):
        for h in range(Hq):
            g = h // 2
            one = O.ds_decode_head(q[b, h], K[b, g, :seq[b]], V[b, g, :seq[b]], lab[b, g, :seq[b]], C[g], k)
            assert np.array_equal(r["idx"][(b, h)], one["idx"])
            assert np.array_equal(r["out"][b, h], one["out"])
            assert r["idx"][(b, h)].max() < seq[b]


PINS = [pin_golden, pin_full_attention, pin_selected_subset_attention, pin_k1_is_argmax_value_row,
        pin_selection_brute_force, pin_score_order, pin_label_and_calibration, pin_batch_gqa_layout]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_ds_pin(pin):
    pin()


# ------------------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# ------------------------------------------------------------------------------------


def _scores_full_key(q, label, channels):
    # uses every label channel against q's leading channels (C ignored)
    lab = np.asarray(label, dtype=np.float32)
    qc = np.asarray(q, dtype=np.float32)[: lab.shape[1]]
    return (lab.astype(np.float64) @ qc.astype(np.float64)).astype(np.float32)


def _select_abs(scores, k):
    return D._topk_desc_ties_low(np.abs(np.asarray(scores, dtype=np.float32)), k)


def _select_lowest(scores, k):
    return D._topk_desc_ties_low(-np.asarray(scores, dtype=np.float32), k)


def _select_ties_high(scores, k):
    s = np.asarray(scores, dtype=np.float64)
    n = s.shape[0]
    order = np.lexsort((-np.arange(n), -s))
    return np.sort(order[: max(0, min(k, n))]).astype(np.int32)


def _attention_no_scale(q, K, V, idx, scale=None):
    return D.__dict__["_orig_ds_attention"](q, K, V, idx, 1.0 if scale is None else scale)


def _attention_all_tokens(q, K, V, idx, scale=None):
    return D.__dict__["_orig_ds_attention"](q, K, V, np.arange(np.asarray(K).shape[0]), scale)


def _scores_exact_sum(q, label, channels):
    qc = np.asarray(q, dtype=np.float64)[np.asarray(channels, dtype=np.int64)]
    return (np.asarray(label, dtype=np.float64) @ qc).astype(np.float32)


def _calibrate_signed(K, r, absmean=None):
    a = np.asarray(K, dtype=np.float64).mean(axis=0) if absmean is None else absmean
    return D._topk_desc_ties_low(a, r)


MUTATIONS = {
    "scores_ignore_channels": ("ds_scores", _scores_full_key),
    "select_by_abs": ("ds_select_tokens", _select_abs),
    "select_lowest": ("ds_select_tokens", _select_lowest),
    "select_ties_high": ("ds_select_tokens", _select_ties_high),
    "attention_no_scale": ("ds_attention", _attention_no_scale),
    "attention_all_tokens": ("ds_attention", _attention_all_tokens),
    "scores_exact_sum": ("ds_scores", _scores_exact_sum),
    "calibrate_signed_mean": ("ds_calibrate_channels", _calibrate_signed),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_ds_mutation_caught(name, monkeypatch):
    fn_name, bad = MUTATIONS[name]
    monkeypatch.setitem(D.__dict__, "_orig_ds_attention", D.ds_attention)
    monkeypatch.setattr(D, fn_name, bad)
    monkeypatch.setattr(O, fn_name, bad)
    failed = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
