"""GPU parity of Double Sparsity decode attention ("大模型DoubleSparse稀疏化技术原理",
sections 离线校准 and 在线前向计算) against the CPU oracle.

* The channel means of the K-outlier calibration agree with the float64 oracle to
  float32 rounding, and the chosen channels equal the oracle's choice on the GPU's means
  (the decision taken on the same numbers).
* The label cache is an exact gather.
* The approximate scores are bit-exact (both sides round each product and add in
  channel order in float32), so the kept tokens are bit-exact too.
* The attention output agrees with the float64 oracle on the same kept tokens to float32
  accumulation error: relative L2 <= 1e-5 per head.

Shapes span grouped queries, ragged sequence lengths, k >= T, k = 1, many tied scores,
float32 caches, head dims 32 to 256, a zero-length sequence and the 16 K-token limit.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle as O
import synth
import free_activation_sparse_b200 as W
from tests.gpu_util import dev_bf16, dev_f32, dev_i32, host, rel_l2, status_word, torch

pytestmark = pytest.mark.gpu

TOL = 1e-5


def _upload(cfg, f32=False):
    if f32:
        cv = lambda bits: dev_f32(synth.f32_from_bf16_bits(bits))  # noqa: E731
    else:
        cv = dev_bf16
    return cv(cfg["q"]), cv(cfg["K"]), cv(cfg["V"])


def _check_decode(cfg, channels, k, f32=False, heads=None):
    q, K, V = _upload(cfg, f32)
    seq = dev_i32(cfg["seq_len"])
    C = dev_i32(channels)
    label = W.ds_label_build(K, seq, C)
    out, idx, sc = W.ds_decode_attention(q, K, V, label, C, seq, k, want_idx=True, want_scores=True)
    out, idx, sc = host(out), host(idx), host(sc)
    qf, Kf, Vf = (synth.f32_from_bf16_bits(cfg[n]) for n in ("q", "K", "V"))
    B, Hq = qf.shape[:2]
    grp = Hq // cfg["Hkv"]
    for b in range(B):
        T = int(cfg["seq_len"][b])
        for h in range(Hq) if heads is None else heads:
            g = h // grp
            lab = O.ds_label_cache(Kf[b, g, :T], channels[g])
            s = O.ds_scores(qf[b, h], lab, channels[g])
            assert np.array_equal(sc[b, h, :T].view(np.uint32), s.view(np.uint32)), (b, h)
            want_idx = O.ds_select_tokens(s, k)
            kk = min(k, T)
            assert np.array_equal(idx[b, h, :kk], want_idx), (b, h)
            want = O.ds_attention(qf[b, h], Kf[b, g, :T], Vf[b, g, :T], want_idx)
            assert rel_l2(out[b, h], want) <= TOL, (b, h, rel_l2(out[b, h], want))
    return out, idx


def test_channel_calibration_and_label_cache():
    cfg = synth.make_ds_decode(seed=31, batch=2, hq=4, hkv=4, seq=[300, 123], dh=64, n_outlier=8)
    _, K, _ = _upload(cfg)
    seq = dev_i32(cfg["seq_len"])
    a = host(W.ds_channel_absmean(K, seq))
    Kf = synth.f32_from_bf16_bits(cfg["K"])
    for g in range(4):
        toks = np.concatenate([Kf[b, g, :int(cfg["seq_len"][b])] for b in range(2)])
        want = O.ds_channel_absmean(toks).astype(np.float32)
        assert np.max(np.abs(a[g] - want) / want) <= 2 ** -23, g
    C = host(W.ds_calibrate_channels(K, seq, 8))
    for g in range(4):
        assert C[g].tolist() == O.ds_calibrate_channels(None, 8, absmean=a[g]).tolist()
        assert C[g].tolist() == cfg["outliers"][g].tolist()  # the planted outliers stand out
    lab = host(W.ds_label_build(K, seq, dev_i32(C)))
    Kb = cfg["K"]
    for b in range(2):
        T = int(cfg["seq_len"][b])
        for g in range(4):
            assert np.array_equal(lab[b, g, :T], Kb[b, g, :T][:, C[g]])
            assert not lab[b, g, T:].any()  # past the sequence: left as it was (zeros)
    # a decode step appends one token's labels
    lab2 = W.ds_label_build(K, seq, dev_i32(C), t0=100, t1=101,
                            label=torch().zeros((2, 4, 300, 8), dtype=torch().bfloat16, device="cuda"))
    lab2 = host(lab2)
    assert np.array_equal(lab2[:, :, 100], lab[:, :, 100])
    assert not lab2[:, :, :100].any() and not lab2[:, :, 101:].any()


@pytest.mark.parametrize("B,hq,hkv,seq,dh,r,k", [
    (1, 4, 4, [1000], 128, 16, 64),
    (2, 8, 2, [777, 1500], 64, 8, 100),
    (3, 2, 1, [1, 5, 4096], 128, 16, 256),
    (1, 2, 2, [1000], 128, 16, 2000),   # k > T: every token
    (2, 4, 4, [513, 64], 128, 16, 1),   # k = 1: the value row of the best token
    (1, 2, 1, [2000], 256, 32, 300),
    (1, 4, 2, [3000], 32, 8, 333),
])
def test_decode_matches_oracle(B, hq, hkv, seq, dh, r, k):
    cfg = synth.make_ds_decode(seed=B * 100 + dh + k, batch=B, hq=hq, hkv=hkv, seq=seq, dh=dh, n_outlier=r,
                               tmax=max(seq) + 7)
    _check_decode(cfg, cfg["outliers"], k)


def test_decode_f32_caches():
    cfg = synth.make_ds_decode(seed=41, batch=2, hq=4, hkv=2, seq=[640, 1000], dh=64, n_outlier=8)
    _check_decode(cfg, cfg["outliers"], 90, f32=True)


def test_decode_many_tied_scores():
    """Label values from {-1, 0, 1}: most scores tie, the kept set goes to lower tokens."""
    cfg = synth.make_ds_decode(seed=42, batch=1, hq=2, hkv=2, seq=[2048], dh=64, n_outlier=8)
    Kf = synth.f32_from_bf16_bits(cfg["K"])
    cfg["K"] = synth.bf16_bits_from_f32(np.clip(np.round(Kf), -1, 1).astype(np.float32))
    qf = synth.f32_from_bf16_bits(cfg["q"])
    cfg["q"] = synth.bf16_bits_from_f32(np.sign(qf).astype(np.float32))
    _check_decode(cfg, cfg["outliers"], 500)


def test_decode_all_channels_is_softmax_attention():
    """Every channel important and k = T: plain attention over all tokens (the float64
    oracle's attention; the oracle's pin ties it to scaled_dot_product_attention)."""
    cfg = synth.make_ds_decode(seed=43, batch=1, hq=2, hkv=2, seq=[900], dh=64, n_outlier=4)
    C = np.tile(np.arange(64, dtype=np.int32), (2, 1))
    out, idx = _check_decode(cfg, C, 900)
    assert np.array_equal(idx[0, 0], np.arange(900))


def test_decode_zero_and_out_of_range_lengths():
    cfg = synth.make_ds_decode(seed=44, batch=3, hq=2, hkv=2, seq=[0, 50, 50], dh=64, n_outlier=8, tmax=64)
    q, K, V = _upload(cfg)
    C = dev_i32(cfg["outliers"])
    good = dev_i32(np.array([0, 50, 64], dtype=np.int32))
    label = W.ds_label_build(K, good, C)
    st = status_word()
    out, _, _ = W.ds_decode_attention(q, K, V, label, C, good, 16, status=st)
    assert int(host(st)[0]) == 0
    assert not host(out)[0].any()  # an empty sequence attends to nothing
    bad = dev_i32(np.array([0, 50, 65], dtype=np.int32))  # beyond Tmax: reported, clamped to 64
    out2, _, _ = W.ds_decode_attention(q, K, V, label, C, bad, 16, status=st)
    assert int(host(st)[0]) == W.ERR_INVALID_ARG
    assert np.array_equal(host(out2), host(out))


def test_decode_long_context_and_repeatable():
    cfg = synth.make_ds_decode(seed=45, batch=1, hq=2, hkv=1, seq=[16384], dh=128, n_outlier=16)
    out1, _ = _check_decode(cfg, cfg["outliers"], 1024)
    q, K, V = _upload(cfg)
    seq = dev_i32(cfg["seq_len"])
    C = dev_i32(cfg["outliers"])
    label = W.ds_label_build(K, seq, C)
    a = host(W.ds_decode_attention(q, K, V, label, C, seq, 1024)[0])
    b = host(W.ds_decode_attention(q, K, V, label, C, seq, 1024)[0])
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(a.view(np.uint32), out1.view(np.uint32))


def test_llama2_7b_workload_sampled_heads():
    """The benchmark's workload (32 heads, 4096 tokens, 16 channels, 256 tokens kept):
    every head's kept set and sampled heads' outputs against the oracle."""
    cfg = synth.make_ds_decode()
    _check_decode(cfg, cfg["outliers"], 256, heads=[0, 7, 31])
