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
import oracle as O
import synth
from tests.gpu_util import dev_bf16, dev_f32, dev_i32, host, rel_l2, status_word, torch

pytestmark = pytest.mark.gpu

TOL = 1e-5  # the same relative L2 bound the other single-token product tests use


def _call_noalloc(Wt, idx, xs, k, B, ld, y, st, count=None, expect=None):
    """Straight through the C ABI (no binding helper)."""
    t = torch()
    code = W.lib.sparse_matvec_noalloc(
        ctypes.c_void_p(Wt.data_ptr()), W.BF16 if Wt.dtype == t.bfloat16 else W.F32, Wt.shape[0], Wt.shape[1],
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(xs.data_ptr()), k,
        None if count is None else ctypes.c_void_p(count.data_ptr()), ld, B,
        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(st.data_ptr()),
        ctypes.c_void_p(t.cuda.current_stream().cuda_stream))
    assert code == (W.OK if expect is None else expect), W.lib.wina_status_string(code)


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
        # and against the float64 oracle on sampled outputs (rows of W)
        rows = np.sort(rng.choice(m, size=64, replace=False))
        Wrows = O.widen_bf16(bits[rows])
        for b in range(B):
            ref = O.sparse_matvec_rows(Wrows, idx[b], xs[b])
            assert rel_l2(got[b][rows], ref) <= TOL, (call, b)


def test_noalloc_per_token_counts():
    """k = -1: each token's count comes from a device array; counts above ld are clamped."""
    t = torch()
    rng = np.random.default_rng(7)
    m, n, ld, B = 4096, 11008, 600, 5
    bits = synth.make_weight(rng, m, n, 0.02, "bf16")
    Wt = W.pack_in_major(dev_bf16(bits))
    idx = np.stack([np.sort(rng.choice(n, size=ld, replace=False)) for _ in range(B)]).astype(np.int32)
    xs = rng.laplace(size=(B, ld)).astype(np.float32)
    cnt = np.array([0, 17, ld, ld + 40, 333], dtype=np.int32)
    di, dx, dc = dev_i32(idx), dev_f32(xs), dev_i32(cnt)
    for call in range(2):
        want = host(W.sparse_matvec(Wt, di, dx, count=dc))
        y = t.full((B, m), float("nan"), dtype=t.float32, device="cuda")
        st = status_word()
        _call_noalloc(Wt, di, dx, -1, B, ld, y, st, count=dc)
        t.cuda.synchronize()
        assert int(host(st)[0]) == 0
        got = host(y)
        for b in range(B):
            kb = min(int(cnt[b]), ld)
            assert rel_l2(got[b], want[b]) <= TOL, (call, b)
            ref = O.sparse_matvec(O.widen_bf16(bits), idx[b][:kb], xs[b][:kb])
            assert rel_l2(got[b], ref) <= TOL, (call, b)
        assert not got[0].any()  # count 0 gives y = 0


def test_noalloc_one_cta_per_token_needs_no_scratch():
    """batch at least the co-resident grid: one CTA per token writes y directly, so
    sizes past the fixed array's limit are accepted (here batch * m = 300 * 11008)."""
    t = torch()
    rng = np.random.default_rng(8)
    m, n, k, B = 11008, 512, 24, 300
    bits = synth.make_weight(rng, m, n, 0.02, "bf16")
    Wt = W.pack_in_major(dev_bf16(bits))
    idx = np.stack([np.sort(rng.choice(n, size=k, replace=False)) for _ in range(B)]).astype(np.int32)
    xs = rng.laplace(size=(B, k)).astype(np.float32)
    di, dx = dev_i32(idx), dev_f32(xs)
    for call in range(2):
        want = host(W.sparse_matvec(Wt, di, dx))
        y = t.full((B, m), float("nan"), dtype=t.float32, device="cuda")
        st = status_word()
        _call_noalloc(Wt, di, dx, k, B, k, y, st)
        t.cuda.synchronize()
        assert int(host(st)[0]) == 0
        got = host(y)
        for b in (0, 1, 150, 299):
            assert rel_l2(got[b], want[b]) <= TOL, (call, b)


def test_noalloc_out_of_range_index_is_reported():
    """An index >= n is never read: the row is skipped and WINA_ERR_INVALID_ARG lands in
    the status word; y stays finite."""
    t = torch()
    rng = np.random.default_rng(9)
    m, n, k = 2048, 1024, 64
    bits = synth.make_weight(rng, m, n, 0.02, "bf16")
    Wt = W.pack_in_major(dev_bf16(bits))
    idx = np.sort(rng.choice(n, size=k, replace=False)).astype(np.int32)[None, :]
    idx[0, 10] = n + 5
    xs = rng.laplace(size=(1, k)).astype(np.float32)
    y = t.full((1, m), float("nan"), dtype=t.float32, device="cuda")
    st = status_word()
    _call_noalloc(Wt, dev_i32(idx), dev_f32(xs), k, 1, k, y, st)
    t.cuda.synchronize()
    assert int(host(st)[0]) == W.ERR_INVALID_ARG
    got = host(y)[0]
    assert np.isfinite(got).all()
    keep = np.ones(k, dtype=bool)
    keep[10] = False
    ref = O.sparse_matvec(O.widen_bf16(bits), idx[0][keep], xs[0][keep])
    assert rel_l2(got, ref) <= TOL


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
