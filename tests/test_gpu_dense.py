"""GPU parity of the dense comparator (every channel kept, output-major weights) against the
float64 CPU oracle: the dense layer and the dense SwiGLU FFN (the FFN with K = n on every
projection). Float32 accumulation of exact bf16 products: relative L2 <= 1e-5.

Shapes cover rows that end in a partial 512-byte slab, fewer rows than warps (each row
then has a warp of its own), rows split between two warps, and rows too long to stage x
in shared memory (the warp-per-row kernel)."""

from __future__ import annotations

import numpy as np
import pytest

import oracle as O
import synth
import free_activation_sparse_b200 as W
from tests.gpu_util import dev_bf16, dev_f32, host, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,n,dt", [(11008, 4096, "bf16"), (4096, 11008, "bf16"), (100, 64, "bf16"),
                                    (512, 256, "f32"), (33, 12, "f32"), (9216, 2304, "bf16"),
                                    (3001, 2312, "bf16"), (777, 1204, "f32"), (40, 32768, "bf16"),
                                    (30, 30000, "f32")])
def test_dense_matvec(m, n, dt):
    rng = np.random.default_rng(m + n)
    Wm = synth.make_weight(rng, m, n, 0.02, dt)
    x = rng.laplace(size=n).astype(np.float32)
    Wd = dev_bf16(Wm) if dt == "bf16" else dev_f32(Wm)
    Wf = O.widen_bf16(Wm) if dt == "bf16" else Wm.astype(np.float64)
    y = host(W.dense_matvec(Wd, dev_f32(x)))
    assert rel_l2(y, O.dense_matvec(Wf, x)) <= 1e-5


@pytest.mark.parametrize("d,ffn", [(4096, 11008), (512, 1536)])
def test_dense_ffn(d, ffn):
    rng = np.random.default_rng(d + ffn)
    Wg = synth.make_weight(rng, ffn, d, 0.02, "bf16")
    Wu = synth.make_weight(rng, ffn, d, 0.02, "bf16")
    Wdn = synth.make_weight(rng, d, ffn, 0.02, "bf16")
    xb = synth.bf16_bits_from_f32(rng.laplace(size=d).astype(np.float32))
    y = host(W.dense_ffn_swiglu(dev_bf16(Wg), dev_bf16(Wu), dev_bf16(Wdn), dev_bf16(xb)))
    Wgf, Wuf, Wdf = (O.widen_bf16(a) for a in (Wg, Wu, Wdn))
    ones_d, ones_f = np.ones(d, dtype=np.float32), np.ones(ffn, dtype=np.float32)
    ref = O.ffn_swiglu(Wgf, Wuf, Wdf, ones_d, ones_d, ones_f, synth.f32_from_bf16_bits(xb), d, d, ffn)
    assert rel_l2(y, ref["y"]) <= 1e-5


def test_dense_matvec_is_repeatable():
    """Rows split between two warps are completed by two atomic adds onto zero, which give
    the same bits in either order: two calls agree bit for bit."""
    rng = np.random.default_rng(5)
    Wm = synth.make_weight(rng, 5000, 2304, 0.02, "bf16")
    Wd, x = dev_bf16(Wm), dev_f32(rng.laplace(size=2304).astype(np.float32))
    a = host(W.dense_matvec(Wd, x))
    b = host(W.dense_matvec(Wd, x))
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("d,ffn,dt", [(2304, 9216, "bf16"), (520, 1032, "bf16"), (256, 700, "f32")])
def test_dense_ffn_shapes(d, ffn, dt):
    rng = np.random.default_rng(d * 3 + ffn)
    Wg, Wu = (synth.make_weight(rng, ffn, d, 0.02, dt) for _ in range(2))
    Wdn = synth.make_weight(rng, d, ffn, 0.02, dt)
    x = rng.laplace(size=d).astype(np.float32)
    dev = dev_bf16 if dt == "bf16" else dev_f32
    y = host(W.dense_ffn_swiglu(dev(Wg), dev(Wu), dev(Wdn), dev_f32(x)))
    wide = O.widen_bf16 if dt == "bf16" else (lambda a: a.astype(np.float64))
    ones_d, ones_f = np.ones(d, dtype=np.float32), np.ones(ffn, dtype=np.float32)
    ref = O.ffn_swiglu(wide(Wg), wide(Wu), wide(Wdn), ones_d, ones_d, ones_f, x, d, d, ffn)
    assert rel_l2(y, ref["y"]) <= 1e-5


def test_dense_ffn_repeat_on_one_workspace():
    """Calls on one workspace alternate between its two g/u copies (each call zeroes the
    other): three calls give the same bits, and a call with other inputs in between does
    not leak into the next."""
    rng = np.random.default_rng(9)
    d, ffn = 1024, 2816
    Wg, Wu = (synth.make_weight(rng, ffn, d, 0.02, "bf16") for _ in range(2))
    Wdn = synth.make_weight(rng, d, ffn, 0.02, "bf16")
    mats = [dev_bf16(a) for a in (Wg, Wu, Wdn)]
    x1 = dev_f32(rng.laplace(size=d).astype(np.float32))
    x2 = dev_f32(rng.laplace(size=d).astype(np.float32))
    ws = W.Workspace(W.OP_DENSE_FFN, d, ffn, 0, 1)
    a = host(W.dense_ffn_swiglu(*mats, x1, ws=ws))
    b = host(W.dense_ffn_swiglu(*mats, x1, ws=ws))
    host(W.dense_ffn_swiglu(*mats, x2, ws=ws))
    c = host(W.dense_ffn_swiglu(*mats, x1, ws=ws))
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(a.view(np.uint32), c.view(np.uint32))
