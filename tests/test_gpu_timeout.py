"""The bounded waits of the single-token FFN kernel give up and report instead of hanging.

The kernel's grid barriers count arrivals in a workspace counter that must start at a
multiple of the grid size (a zero-filled workspace). Starting it at 1 makes one CTA's
target unreachable: that CTA's wait runs out, it records WINA_ERR_TIMEOUT and returns;
the other CTAs then wait in vain at the next barrier and give up the same way. With the
wait limit shortened to 1 ms (wina_set_wait_limit_ns), the call completes at once with
the status set; after the workspace is zero-filled again, the same call succeeds. No
fault, trap or endless loop is involved: the failure is a counter value the host wrote.
"""

from __future__ import annotations

import time

import numpy as np
import pytest

import oracle as O
import synth
import free_activation_sparse_b200 as W
from tests.gpu_util import dev_bf16, host, rel_l2, status_word, torch

pytestmark = pytest.mark.gpu


def test_barrier_wait_runs_out_and_reports():
    t = torch()
    rng = np.random.default_rng(21)
    d, ffn = 1024, 2816
    Wg = synth.make_weight(rng, ffn, d, 0.02, "bf16")
    Wu = synth.make_weight(rng, ffn, d, 0.02, "bf16")
    Wd = synth.make_weight(rng, d, ffn, 0.02, "bf16")
    f = W.ffn_prepare(dev_bf16(Wg), dev_bf16(Wu), dev_bf16(Wd))
    xb = synth.bf16_bits_from_f32(rng.laplace(size=(1, d)).astype(np.float32))
    x = dev_bf16(xb)
    kg, kd = d // 2, ffn // 2
    ws = W.Workspace(W.OP_FFN_SWIGLU, d, ffn, 0, 1)
    st = status_word()
    try:
        W.lib.wina_set_wait_limit_ns(1_000_000)  # 1 ms
        ws.buf[8:16].view(t.int64)[0] = 1  # the barrier's arrival counter, off by one
        t.cuda.synchronize()
        t0 = time.perf_counter()
        W.sparse_ffn_swiglu(f, x, W.GATE_TOPK, kg, kg, kd, ws=ws, status=st)
        t.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        assert int(host(st)[0]) == W.ERR_TIMEOUT
        assert elapsed < 5.0
    finally:
        W.lib.wina_set_wait_limit_ns(0)
    ws.buf.zero_()
    st.zero_()
    y = host(W.sparse_ffn_swiglu(f, x, W.GATE_TOPK, kg, kg, kd, ws=ws, status=st))
    assert int(host(st)[0]) == 0
    Wgf, Wuf, Wdf = (O.widen_bf16(a) for a in (Wg, Wu, Wd))
    cg, cu, cd = (host(c) for c in (f.c_gate, f.c_up, f.c_down))
    ref = O.ffn_swiglu(Wgf, Wuf, Wdf, cg, cu, cd, synth.f32_from_bf16_bits(xb)[0], kg, kg, kd)
    assert rel_l2(y[0], ref["y"]) <= 5e-3


def test_dense_ffn_barrier_wait_runs_out_and_reports():
    """The same for the dense comparator's cooperative kernel (its barrier counter leads
    its workspace)."""
    t = torch()
    rng = np.random.default_rng(22)
    d, ffn = 512, 1536
    Wg = synth.make_weight(rng, ffn, d, 0.02, "bf16")
    Wu = synth.make_weight(rng, ffn, d, 0.02, "bf16")
    Wd = synth.make_weight(rng, d, ffn, 0.02, "bf16")
    xb = synth.bf16_bits_from_f32(rng.laplace(size=d).astype(np.float32))
    args = (dev_bf16(Wg), dev_bf16(Wu), dev_bf16(Wd), dev_bf16(xb))
    ws = W.Workspace(W.OP_DENSE_FFN, d, ffn, 0, 1)
    st = status_word()
    try:
        W.lib.wina_set_wait_limit_ns(1_000_000)  # 1 ms
        ws.buf[8:16].view(t.int64)[0] = 1  # the barrier's arrival counter, off by one
        t.cuda.synchronize()
        t0 = time.perf_counter()
        W.dense_ffn_swiglu(*args, ws=ws, status=st)
        t.cuda.synchronize()
        assert int(host(st)[0]) == W.ERR_TIMEOUT
        assert time.perf_counter() - t0 < 5.0
    finally:
        W.lib.wina_set_wait_limit_ns(0)
    ws.buf.zero_()
    st.zero_()
    y = host(W.dense_ffn_swiglu(*args, ws=ws, status=st))
    assert int(host(st)[0]) == 0
    ones_d, ones_f = np.ones(d, dtype=np.float32), np.ones(ffn, dtype=np.float32)
    ref = O.ffn_swiglu(*(O.widen_bf16(a) for a in (Wg, Wu, Wd)), ones_d, ones_d, ones_f,
                       synth.f32_from_bf16_bits(xb), d, d, ffn)
    assert rel_l2(y, ref["y"]) <= 1e-5
