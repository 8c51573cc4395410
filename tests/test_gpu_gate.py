"""GPU parity of the offline preparation and the per-token gates against the CPU oracle.

Index sets must match bit-exactly (given the same float32 scores); column norms and
packed weights must match bit-exactly.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle as O
import synth
import free_activation_sparse_b200 as W
from tests.gpu_util import dev_bf16, dev_f32, host, status_word, torch

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------------------
# a0: packing and column norms
# ------------------------------------------------------------------------------------


@pytest.mark.parametrize("m,n", [(1, 1), (37, 53), (512, 256), (33, 4096)])
def test_pack_in_major_bit_exact(m, n):
    rng = np.random.default_rng(m * 1000 + n)
    bits = synth.make_weight(rng, m, n, 0.02, "bf16")
    Wt = W.pack_in_major(dev_bf16(bits))
    assert np.array_equal(host(Wt), bits.T)
    f = synth.make_weight(rng, m, n, 1.0, "f32")
    assert np.array_equal(host(W.pack_in_major(dev_f32(f))), f.T)


def test_col_norms_bit_exact_fp32_linear():
    cfg = synth.make_linear_512x256_f32()
    Wd = dev_f32(cfg["W"])
    want = O.col_norms(cfg["W"])
    assert np.array_equal(host(W.col_norms(Wd)), want)
    assert np.array_equal(host(W.col_norms(W.pack_in_major(Wd), layout="in_major")), want)


@pytest.mark.parametrize("m,n", [(11008, 4096), (4096, 11008), (3, 5), (100, 257)])
def test_col_norms_bit_exact_bf16(m, n):
    rng = np.random.default_rng(n)
    bits = synth.make_weight(rng, m, n, 0.02, "bf16")
    want = O.col_norms(O.widen_bf16(bits))
    Wd = dev_bf16(bits)
    got = host(W.col_norms(Wd))
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} columns differ, e.g. {bad[:5]}"
    assert np.array_equal(host(W.col_norms(W.pack_in_major(Wd), layout="in_major")), want)


# ------------------------------------------------------------------------------------
# a1 + a2: scores and exact top-K
# ------------------------------------------------------------------------------------


def _check_select(x_dev, x_vals_f32, c_np, k, B):
    c_dev = dev_f32(c_np) if c_np is not None else None
    idx, xs, sc = W.select_topk(x_dev, c_dev, k, want_scores=True)
    idx, xs, sc = host(idx), host(xs), host(sc)
    for b in range(B):
        want_sc = O.gate_scores(x_vals_f32[b], c_np)
        assert np.array_equal(sc[b], want_sc)
        want = O.select_topk(want_sc, k)
        assert np.array_equal(idx[b], want), f"token {b}: {np.setxor1d(idx[b], want)[:8]}"
        assert np.array_equal(xs[b], x_vals_f32[b][want])


def test_select_linear_512x256():
    cfg = synth.make_linear_512x256_f32()
    c = O.col_norms(cfg["W"])
    _check_select(dev_f32(cfg["x"]), cfg["x"], c, 128, 1)


@pytest.mark.parametrize("n,k", [(4096, 2048), (4096, 1434), (11008, 5504), (11008, 3853), (14336, 143)])
def test_select_llama_shapes(n, k):
    rng = np.random.default_rng(n + k)
    B = 3
    x = synth.bf16_bits_from_f32(rng.laplace(size=(B, n)).astype(np.float32))
    c = (0.02 * rng.lognormal(0, 0.5, n) * np.sqrt(4096)).astype(np.float32)
    _check_select(dev_bf16(x), synth.f32_from_bf16_bits(x), c, k, B)


@pytest.mark.parametrize("n", [1, 2, 31, 33, 1000, 4097, 32768])
def test_select_ragged_and_extreme_k(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal((2, n)).astype(np.float32)
    c = rng.lognormal(0, 0.5, n).astype(np.float32)
    for k in sorted({0, 1, n // 2, max(n - 1, 0), n}):
        _check_select(dev_f32(x), x, c, k, 2)


def test_select_ties_go_to_lower_index():
    rng = np.random.default_rng(0)
    n = 5000
    # a tiny alphabet of values: thousands of exact ties at every boundary
    x = rng.integers(-3, 4, size=(4, n)).astype(np.float32)
    for c in (None, np.ones(n, dtype=np.float32), np.full(n, 0.5, dtype=np.float32)):
        for k in (1, 7, 2500, 4999):
            _check_select(dev_f32(x), x, c, k, 4)
    z = np.zeros((1, n), dtype=np.float32)  # all scores zero: the first k channels
    _check_select(dev_f32(z), z, np.ones(n, dtype=np.float32), 123, 1)


def test_select_teal_gate_recovers_nonzeros():
    cfg = synth.make_ultrasparse_down(batch=8)
    xv = synth.f32_from_bf16_bits(cfg["x"])
    idx, _ = W.select_topk(dev_bf16(cfg["x"]), None, cfg["nnz"])
    idx = host(idx)
    for b in range(8):
        assert np.array_equal(idx[b], np.nonzero(xv[b])[0])


# ------------------------------------------------------------------------------------
# a2': the Spark statistical threshold
# ------------------------------------------------------------------------------------


def _check_stat(v_dev, v_vals, s, cap=None):
    B, n = v_vals.shape
    idx, xs, count, t = W.stat_topk_threshold(v_dev, s, cap=cap)
    idx, xs, count, t = host(idx), host(xs), host(count), host(t)
    for b in range(B):
        ref = O.spark_threshold(v_vals[b], s)
        sig = ref["sigma"]
        assert abs(float(t[b]) - ref["t"]) <= 1e-5 * sig + 1e-6 * abs(ref["t"])
        kept = idx[b][: min(count[b], idx.shape[1])]
        # the GPU's set is exactly the upper level set of its own threshold
        # (compared in float64 against the float64 t it used: recover it from count)
        assert np.all(np.diff(kept) > 0)
        diff = np.setxor1d(kept, ref["idx"]) if cap is None else np.array([], dtype=np.int64)
        if diff.size:
            assert np.all(np.abs(v_vals[b][diff].astype(np.float64) - ref["t"]) <= 1e-5 * sig)
        if cap is None:
            assert count[b] == kept.size
            assert np.array_equal(xs[b][: kept.size], v_vals[b][kept])
    return idx, count


def test_stat_gemma_shapes_batch64():
    cfg = synth.make_gemma2_2b_spark(batch=64, weights=False)
    _check_stat(dev_f32(cfg["x"]), cfg["x"], cfg["s"])
    _check_stat(dev_f32(cfg["v"]), cfg["v"], cfg["s"])
    _check_stat(dev_bf16(cfg["x_bf16"]), synth.f32_from_bf16_bits(cfg["x_bf16"]), cfg["s"])


def test_stat_keep_fraction_and_overlap_with_exact_topk():
    cfg = synth.make_gemma2_2b_spark(batch=64, weights=False)
    for vec, k in ((cfg["x"], cfg["k_d"]), (cfg["v"], cfg["k_ffn"])):
        idx, count = _check_stat(dev_f32(vec), vec, cfg["s"])
        n = vec.shape[1]
        fr = count / n
        assert abs(fr.mean() - cfg["s"]) < 0.01
        for b in range(vec.shape[0]):
            S = idx[b][: count[b]]
            T = O.exact_topk_signed(vec[b], k)
            ov = O.overlap(S, T)
            assert ov["inter"] == min(len(S), k)  # nested upper level sets


def test_stat_capacity_overflow_sets_status():
    rng = np.random.default_rng(1)
    v = rng.standard_normal((3, 4096)).astype(np.float32)
    st = status_word()
    idx, xs, count, t = W.stat_topk_threshold(dev_f32(v), 0.3, cap=100, status=st)
    count = host(count)
    assert np.all(count > 100)
    assert int(host(st)[0]) == W.ERR_CAPACITY
    idx = host(idx)
    for b in range(3):
        ref = O.spark_threshold(v[b], 0.3)["idx"]
        assert np.array_equal(idx[b], ref[:100])


def test_stat_degenerate_constant_vector():
    v = np.full((2, 777), 0.25, dtype=np.float32)
    idx, xs, count, t = W.stat_topk_threshold(dev_f32(v), 0.5)
    assert host(count).tolist() == [0, 0]
