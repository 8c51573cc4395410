"""The batched FFN path inside a CUDA graph: the up projection runs on the library's side
stream, forked from and joined back to the caller's stream by events, so a capture of the
caller's stream must hold both branches. A captured call, replayed on new inputs, must
give the kept sets of an eager call and the oracle's y (the union product adds its K
split with float atomics, so y is compared within the union tests' float32 bound)."""

from __future__ import annotations

import numpy as np
import pytest

import oracle as O
import synth
import free_activation_sparse_b200 as W
from tests.gpu_util import dev_bf16, host, rel_l2, status_word, torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["topk", "stat"])
def test_batched_ffn_graph_replay_matches_eager_and_oracle(mode):
    t = torch()
    rng = np.random.default_rng(31)
    d, ffn, B = 1024, 2816, 8
    Wg = synth.make_weight(rng, ffn, d, 0.02, "bf16")
    Wu = synth.make_weight(rng, ffn, d, 0.02, "bf16")
    Wd = synth.make_weight(rng, d, ffn, 0.02, "bf16")
    f = W.ffn_prepare(dev_bf16(Wg), dev_bf16(Wu), dev_bf16(Wd))
    xa = synth.bf16_bits_from_f32(rng.laplace(size=(B, d)).astype(np.float32))
    xb = synth.bf16_bits_from_f32(rng.laplace(size=(B, d)).astype(np.float32))
    x = dev_bf16(xa)
    kg, kd = d // 2, ffn // 2
    ws = W.Workspace(W.OP_FFN_SWIGLU, d, ffn, 0, B)
    st = status_word()
    y = t.empty((B, d), dtype=t.float32, device="cuda")

    def call():
        if mode == "topk":
            W.sparse_ffn_swiglu(f, x, W.GATE_TOPK, kg, kg, kd, ws=ws, status=st, y=y)
        else:
            W.sparse_ffn_swiglu(f, x, W.GATE_STAT, s=0.3, ws=ws, status=st, y=y)

    call()  # eager first: the side stream exists before the capture
    t.cuda.synchronize()
    g = t.cuda.CUDAGraph()
    side = t.cuda.Stream()
    side.wait_stream(t.cuda.current_stream())
    with t.cuda.stream(side):
        with t.cuda.graph(g, stream=side):
            call()
    t.cuda.synchronize()
    x.copy_(dev_bf16(xb))  # replay on other inputs
    g.replay()
    t.cuda.synchronize()
    assert int(host(st)[0]) == 0
    y_graph = host(y).copy()
    views = W.ffn_ws_view(ws, d, ffn, B)
    kept_graph = {k: host(views[k]).copy() for k in ("keep_gate", "keep_up", "keep_down")}
    h_graph = host(views["h"]).copy()
    call()  # the same inputs, eager
    t.cuda.synchronize()
    views = W.ffn_ws_view(ws, d, ffn, B)
    for k in ("keep_gate", "keep_up", "keep_down"):
        assert np.array_equal(kept_graph[k], host(views[k])), k
    assert rel_l2(y_graph, host(y)) <= 1e-5
    # and the oracle on the replayed inputs (the down set taken on the GPU's h, as in the
    # FFN tests; Spark sets may differ only within 1e-5 sigma of the threshold, where the
    # float64 moments' summation order can decide)
    Wdf = O.widen_bf16(Wd)
    cg, cu, cd = (host(c) for c in (f.c_gate, f.c_up, f.c_down))
    xf = synth.f32_from_bf16_bits(xb)
    for b in range(B):
        gk, uk, dk = (np.nonzero(kept_graph[k][b])[0] for k in ("keep_gate", "keep_up", "keep_down"))
        if mode == "topk":
            assert np.array_equal(gk, O.wina_select(xf[b], cg, kg))
            assert np.array_equal(uk, O.wina_select(xf[b], cu, kg))
            assert np.array_equal(dk, O.wina_select(h_graph[b], cd, kd))
        else:
            for got, v in ((gk, xf[b]), (dk, h_graph[b])):
                ref = O.spark_threshold(v, 0.3)
                diff = np.setxor1d(got, ref["idx"])
                assert np.all(np.abs(v[diff] - ref["t"]) <= 1e-5 * ref["sigma"])
            assert np.array_equal(uk, gk)
        want = O.sparse_matvec(Wdf, dk, h_graph[b][dk].astype(np.float64))
        assert rel_l2(y_graph[b], want) <= 1e-5
