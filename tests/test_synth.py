"""The seeded generators: determinism, bf16 rounding, workload shapes (CPU only)."""

import numpy as np

import synth


def test_bf16_round_nearest_even():
    v = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0], dtype=np.float32)
    bits = synth.bf16_bits_from_f32(v)
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000]
    assert synth.f32_from_bf16_bits(bits).tolist() == [1.0, 1.0, 1.015625, -2.5, 0.0]


def test_keep_counts():
    assert synth.keep_count(0.5, 4096) == 2048
    assert synth.keep_count(0.5, 11008) == 5504
    assert synth.keep_count(0.65, 4096) == 1434
    assert synth.keep_count(0.65, 11008) == 3853
    assert synth.spark_keep_count(0.08, 2304) == 184
    assert synth.spark_keep_count(0.08, 9216) == 737


def test_deterministic_and_shaped():
    a = synth.make_linear_512x256_f32()
    b = synth.make_linear_512x256_f32()
    assert a["W"].shape == (512, 256) and a["W"].dtype == np.float32
    assert a["x"].shape == (1, 256)
    assert np.array_equal(a["W"], b["W"]) and np.array_equal(a["x"], b["x"])
    g = synth.make_gemma2_2b_spark(batch=3, weights=False)
    assert g["x"].shape == (3, 2304) and g["v"].shape == (3, 9216)
    assert g["k_d"] == 184 and g["k_ffn"] == 737


def test_weight_recipe_column_scale():
    rng = np.random.default_rng(0)
    w = synth.make_weight(rng, 4000, 8, 0.02, "f32")
    # per-column std = 0.02 * col_scale: columns differ in scale, rows do not
    col_std = w.std(axis=0)
    assert col_std.max() / col_std.min() > 1.2
    assert w.dtype == np.float32


def test_bench_bytes_per_layer():
    # The bench's unit: the kept rows of the three bf16 weights (Llama-7B FFN, d 4096,
    # ffn 11008) plus the vectors that cross HBM (x bf16, c_gate/c_up/c_down and y float32).
    import bench

    rows_p50 = (2048 + 2048) * 11008 * 2 + 5504 * 4096 * 2
    rows_p65 = (1434 + 1434) * 11008 * 2 + 3853 * 4096 * 2
    assert rows_p50 == 135_266_304 and rows_p65 == 94_705_664
    vecs = 4096 * 2 + 2 * 4096 * 4 + 11008 * 4 + 4096 * 4
    assert bench.layer_bytes(2048, 2048, 5504) == rows_p50 + vecs == 135_367_680
    kg, kd = synth.keep_count(0.65, 4096), synth.keep_count(0.65, 11008)
    assert (kg, kd) == (1434, 3853)
    assert bench.layer_bytes(kg, kg, kd) == rows_p65 + vecs
