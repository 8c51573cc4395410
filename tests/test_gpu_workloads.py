"""Full-size workloads on the GPU, checked against the oracle on sampled outputs (the
oracle computes the sampled output rows one by one) and on exact kept sets:

  * Llama-3-8B-shaped decoder layer (Q, K, V, O, gate, up, down; per-projection
    sparsity from a seeded U(0.4, 0.7) schedule), batch 1, 4 and 16;
  * the ultra-sparse down projection 14336 -> 4096 with 1% nonzero inputs, batch 256.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle as O
import synth
import free_activation_sparse_b200 as W
from tests.gpu_util import dev_bf16, host, rel_l2, status_word

pytestmark = pytest.mark.gpu

N_SAMPLE = 96


@pytest.fixture(scope="module")
def llama3():
    cfg = synth.make_llama3_8b_layer(batch=16)
    dev = {name: dev_bf16(w) for name, w in cfg["W"].items()}
    Wt = {name: W.pack_in_major(w) for name, w in dev.items()}
    c = {name: W.col_norms(w) for name, w in dev.items()}
    return cfg, Wt, c


def _sampled_rows(cfg, name, rng):
    m = cfg["shape"][name][0]
    rows = np.sort(rng.choice(m, size=min(N_SAMPLE, m), replace=False))
    return rows, O.widen_bf16(cfg["W"][name][rows])


@pytest.mark.parametrize("B", [1, 4, 16])
def test_llama3_attention_projections(llama3, B):
    cfg, Wt, c = llama3
    rng = np.random.default_rng(B)
    x32 = synth.f32_from_bf16_bits(cfg["x"][:B])
    o32 = synth.f32_from_bf16_bits(cfg["o_in"][:B])
    for name, xin, xbits in (("q", x32, cfg["x"][:B]), ("k", x32, cfg["x"][:B]), ("v", x32, cfg["x"][:B]),
                             ("o", o32, cfg["o_in"][:B])):
        k = cfg["k"][name]
        cn = host(c[name])
        idx, xs = W.select_topk(dev_bf16(xbits), c[name], k)
        y = host(W.sparse_matvec(Wt[name], idx, xs))
        idx = host(idx)
        rows, Wr = _sampled_rows(cfg, name, rng)
        for b in range(B):
            want = O.wina_select(xin[b], cn, k)
            assert np.array_equal(idx[b], want), name
            assert rel_l2(y[b][rows], O.sparse_matvec_rows(Wr, want, xin[b][want])) <= 1e-5, name


@pytest.mark.parametrize("B", [1, 4, 16])
def test_llama3_ffn(llama3, B):
    cfg, Wt, c = llama3
    rng = np.random.default_rng(100 + B)
    f = W.FfnWeights(Wt["gate"], Wt["up"], Wt["down"], c["gate"], c["up"], c["down"])
    kg, ku, kd = cfg["k"]["gate"], cfg["k"]["up"], cfg["k"]["down"]
    ws = W.Workspace(W.OP_FFN_SWIGLU, 4096, 14336, 0, B)
    st = status_word()
    y = host(W.sparse_ffn_swiglu(f, dev_bf16(cfg["x"][:B]), W.GATE_TOPK, kg, ku, kd, ws=ws, status=st))
    assert int(host(st)[0]) == 0
    v = {k: host(t) for k, t in W.ffn_ws_view(ws, 4096, 14336, B).items()}
    x32 = synth.f32_from_bf16_bits(cfg["x"][:B])
    cg, cu, cd = host(c["gate"]), host(c["up"]), host(c["down"])
    grow, Wgr = _sampled_rows(cfg, "gate", rng)
    urow = grow
    Wur = O.widen_bf16(cfg["W"]["up"][urow])
    drow, Wdr = _sampled_rows(cfg, "down", rng)
    for b in range(B):
        ig = O.wina_select(x32[b], cg, kg)
        iu = O.wina_select(x32[b], cu, ku)
        assert np.array_equal(np.nonzero(v["keep_gate"][b])[0], ig)
        assert np.array_equal(np.nonzero(v["keep_up"][b])[0], iu)
        x64 = x32[b].astype(np.float64)
        h_rows = O.silu(O.sparse_matvec_rows(Wgr, ig, x64[ig])) * O.sparse_matvec_rows(Wur, iu, x64[iu])
        h_gpu = v["h"][b]
        assert rel_l2(h_gpu[grow], h_rows) <= 1e-5
        idn = O.wina_select(h_gpu, cd, kd)
        assert np.array_equal(np.nonzero(v["keep_down"][b])[0], idn)
        assert rel_l2(y[b][drow], O.sparse_matvec_rows(Wdr, idn, h_gpu[idn].astype(np.float64))) <= 1e-5


def test_ultrasparse_down_batch256():
    cfg = synth.make_ultrasparse_down()
    Wd = dev_bf16(cfg["W"])
    Wt = W.pack_in_major(Wd)
    xb = dev_bf16(cfg["x"])
    idx, xs = W.select_topk(xb, None, cfg["nnz"])
    st = status_word()
    y = host(W.sparse_matvec(Wt, idx, xs, status=st))
    assert int(host(st)[0]) == 0
    idx = host(idx)
    x32 = synth.f32_from_bf16_bits(cfg["x"])
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(cfg["m"], size=N_SAMPLE, replace=False))
    Wr = O.widen_bf16(cfg["W"][rows])
    union = O.union_indices([np.nonzero(x32[b])[0] for b in range(x32.shape[0])])
    assert 0.85 < union.size / cfg["n"] < 0.97  # ~92% of columns are touched by some token
    for b in range(x32.shape[0]):
        nz = np.nonzero(x32[b])[0]
        assert np.array_equal(idx[b], nz)
        assert rel_l2(y[b][rows], O.sparse_matvec_rows(Wr, nz, x32[b][nz])) <= 1e-5
