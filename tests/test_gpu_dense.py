"""GPU parity of the dense comparator (every channel kept, output-major weights) against the
float64 CPU oracle: the dense layer and the dense SwiGLU FFN (the FFN with K = n on every
projection). Float32 accumulation of exact bf16 products: relative L2 <= 1e-5."""

from __future__ import annotations

import numpy as np
import pytest

import oracle as O
import synth
import free_activation_sparse_b200 as W
from tests.gpu_util import dev_bf16, dev_f32, host, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,n,dt", [(11008, 4096, "bf16"), (4096, 11008, "bf16"), (100, 64, "bf16"),
                                    (512, 256, "f32"), (33, 12, "f32")])
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
