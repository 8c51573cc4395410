"""sparse_matvec_noalloc: the workspace-free entry point, for callers that cannot
allocate device memory (its scratch is a fixed array the library declares in device
memory). Called through the C ABI and compared with sparse_matvec, which takes a
caller-provided workspace, on two calls in a row (the second reuses the scratch the
first left behind).

This file is collected last on purpose, so that a run that stops at the first failure
has already run every other test.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest

import free_activation_sparse_b200 as W
import synth
from tests.gpu_util import dev_bf16, dev_f32, dev_i32, host, rel_l2, status_word, torch

pytestmark = pytest.mark.gpu

TOL = 1e-5  # the same relative L2 bound the other single-token product tests use


def _call_noalloc(Wt, idx, xs, k, B, ld, y, st):
    """Straight through the C ABI (no binding helper)."""
    t = torch()
    code = W.lib.sparse_matvec_noalloc(
        ctypes.c_void_p(Wt.data_ptr()), W.BF16 if Wt.dtype == t.bfloat16 else W.F32, Wt.shape[0], Wt.shape[1],
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(xs.data_ptr()), k, None, ld, B,
        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(st.data_ptr()),
        ctypes.c_void_p(t.cuda.current_stream().cuda_stream))
    assert code == W.OK, W.lib.wina_status_string(code)


@pytest.mark.parametrize("m,n,k,B", [(11008, 4096, 2048, 1), (4096, 11008, 5504, 1), (4096, 14336, 143, 40),
                                     (1024, 4096, 1500, 3)])
def test_noalloc_matches_workspace_version_twice(m, n, k, B):
    t = torch()
    rng = np.random.default_rng(m + n + k + B)
    bits = synth.make_weight(rng, m, n, 0.02, "bf16")
    Wt = W.pack_in_major(dev_bf16(bits))
    for call in range(2):  # two calls in a row with different inputs
        idx = np.stack([np.sort(rng.choice(n, size=k, replace=False)) for _ in range(B)]).astype(np.int32)
        xs = rng.laplace(size=(B, k)).astype(np.float32)
        di, dx = dev_i32(idx), dev_f32(xs)
        want = host(W.sparse_matvec(Wt, di, dx))
        y = t.full((B, m), float("nan"), dtype=t.float32, device="cuda")
        st = status_word()
        _call_noalloc(Wt, di, dx, k, B, k, y, st)
        t.cuda.synchronize()
        assert int(host(st)[0]) == 0
        got = host(y)
        for b in range(B):
            assert rel_l2(got[b], want[b]) <= TOL, (call, b)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    t = torch()
    Wt = t.zeros((16, 32768), dtype=t.bfloat16, device="cuda")
    idx = t.zeros((64, 4), dtype=t.int32, device="cuda")
    xs = t.zeros((64, 4), dtype=t.float32, device="cuda")
    y = t.empty((64, 32768), dtype=t.float32, device="cuda")
    st = status_word()
    code = W.lib.sparse_matvec_noalloc(ctypes.c_void_p(Wt.data_ptr()), W.BF16, 16, 32768,
                                       ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(xs.data_ptr()), 4, None, 4,
                                       64, ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(st.data_ptr()), None)
    assert code == W.ERR_INVALID_ARG  # 64 * 32768 outputs > 2^20
