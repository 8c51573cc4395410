"""Host-side checks of the C ABI (CPU only, no kernel launches).

The library must load, export every function include/wina.h declares, compute the
normal quantile on the host, size workspaces, and reject bad arguments with the
documented status codes before any CUDA call is made.
"""

from __future__ import annotations

import ctypes
import math
from statistics import NormalDist

import pytest

import free_activation_sparse_b200 as W

FAKE = ctypes.c_void_p(1 << 20)  # a 16-byte-aligned address that is never dereferenced:
MISALIGNED = ctypes.c_void_p((1 << 20) + 2)  # every call below must fail validation first


def test_exports_every_declared_symbol():
    names = W.declared_symbols()
    assert {"wina_select_topk", "stat_topk_threshold", "sparse_matvec", "sparse_ffn_swiglu",
            "wina_col_norms", "wina_pack_in_major", "wina_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(W.lib, n), f"libwina.so does not export {n}"


def test_abi_version_and_strings():
    assert W.abi_version() == 1
    for code in range(7):
        assert W.lib.wina_status_string(code)
    assert W.lib.wina_status_string(99) == b"unknown status"


@pytest.mark.parametrize("p", [1e-12, 1e-6, 0.01, 0.08, 0.3, 0.5, 0.7, 0.92, 0.99, 1 - 1e-6])
def test_normal_quantile_matches_reference(p):
    want = NormalDist().inv_cdf(p)
    got = W.normal_quantile(p)
    assert abs(got - want) <= 1e-12 * max(1.0, abs(want)), (p, got, want)


def test_normal_quantile_domain():
    assert math.isnan(W.normal_quantile(0.0))
    assert math.isnan(W.normal_quantile(1.0))
    assert math.isnan(W.normal_quantile(-0.5))
    assert W.normal_quantile(0.5) == 0.0


def test_workspace_sizes():
    s1 = W.workspace_size(W.OP_SPARSE_MATVEC, 4096, 11008, 2048, 1)
    assert s1 >= 296 * 11008 * 4
    assert W.workspace_size(W.OP_SPARSE_MATVEC, 4096, 11008, 2048, 4096) < s1  # one CTA per token: no partials
    f1 = W.workspace_size(W.OP_FFN_SWIGLU, 4096, 11008, 0, 1)
    assert f1 >= 2 * 296 * 11008 * 4  # the single-token kernel's partial rows (two per CTA)
    f4 = W.workspace_size(W.OP_FFN_SWIGLU, 4096, 11008, 0, 4)
    f8 = W.workspace_size(W.OP_FFN_SWIGLU, 4096, 11008, 0, 8)
    assert f8 > f4 >= 4 * (2 * 4096 + 11008) * 8  # several tokens: per-token index and value lists
    assert W.workspace_size(W.OP_SELECT_TOPK, 10, 10, 1, 1) == 0
    dn = W.workspace_size(W.OP_DENSE_FFN, 4096, 11008, 0, 1)
    assert dn >= 128 + 2 * 11008 * 4  # barrier, g, u
    assert W.workspace_size(W.OP_DENSE_FFN, 4096, 11008, 0, 2) == 0  # one token
    assert W.workspace_size(W.OP_FFN_SWIGLU, 0, 10, 0, 1) == 0


def test_ffn_ws_view_offsets_are_disjoint():
    v = W._FfnView()
    assert W.lib.wina_ffn_ws_view(4096, 11008, 2, ctypes.byref(v)) == W.OK
    spans = sorted([(v.h, 2 * 11008 * 4), (v.keep_gate, 2 * 4096), (v.keep_up, 2 * 4096),
                    (v.keep_down, 2 * 11008), (v.stamps, 16 * 8), (v.cta_t, 296 * 4 * 8)])
    for (a, la), (b, _) in zip(spans, spans[1:]):
        assert a + la <= b
        assert a % 256 == 0
    assert spans[-1][0] + spans[-1][1] <= W.workspace_size(W.OP_FFN_SWIGLU, 4096, 11008, 0, 2)
    assert W.lib.wina_ffn_ws_view(0, 1, 1, ctypes.byref(v)) == W.ERR_INVALID_ARG


def test_select_rejects_bad_arguments():
    L = W.lib
    ok_args = dict(x=FAKE, xdt=W.BF16, c=FAKE, n=4096, k=2048, batch=1, idx=FAKE, xs=FAKE, scores=None)

    def call(**kw):
        a = dict(ok_args, **kw)
        return L.wina_select_topk(a["x"], a["xdt"], a["c"], a["n"], a["k"], a["batch"], a["idx"], a["xs"],
                                  a["scores"], None)

    assert call(xdt=7) == W.ERR_UNSUPPORTED_DTYPE
    assert call(n=0) == W.ERR_INVALID_ARG
    assert call(n=40000) == W.ERR_INVALID_ARG
    assert call(k=4097) == W.ERR_INVALID_ARG
    assert call(k=-1) == W.ERR_INVALID_ARG
    assert call(batch=0) == W.ERR_INVALID_ARG
    assert call(x=None) == W.ERR_INVALID_ARG
    assert call(idx=None) == W.ERR_INVALID_ARG
    assert call(idx=MISALIGNED) == W.ERR_INVALID_ARG


def test_stat_rejects_bad_arguments():
    L = W.lib

    def call(s=0.08, n=9216, cap=9216, count=FAKE, v=FAKE, vdt=W.F32):
        return L.stat_topk_threshold(v, vdt, n, s, 1, FAKE, FAKE, count, FAKE, cap, None, None)

    assert call(s=0.0) == W.ERR_INVALID_ARG
    assert call(s=1.0) == W.ERR_INVALID_ARG
    assert call(s=float("nan")) == W.ERR_INVALID_ARG
    assert call(cap=-1) == W.ERR_INVALID_ARG
    assert call(count=None) == W.ERR_INVALID_ARG
    assert call(n=0) == W.ERR_INVALID_ARG
    assert call(vdt=5) == W.ERR_UNSUPPORTED_DTYPE


def test_sparse_matvec_rejects_bad_arguments():
    L = W.lib
    need = W.workspace_size(W.OP_SPARSE_MATVEC, 4096, 11008, 2048, 1)

    def call(Wt=FAKE, wdt=W.BF16, n=4096, m=11008, k=2048, count=None, ld=2048, batch=1, y=FAKE, ws=FAKE,
             ws_bytes=need):
        return L.sparse_matvec(Wt, wdt, n, m, FAKE, FAKE, k, count, ld, batch, y, ws, ws_bytes, None, None)

    assert call(wdt=9) == W.ERR_UNSUPPORTED_DTYPE
    assert call(m=11004) == W.ERR_INVALID_ARG  # not a multiple of 8 bf16
    assert call(m=40000) == W.ERR_INVALID_ARG  # wider than the kernel's register tile
    assert call(k=2049) == W.ERR_INVALID_ARG
    assert call(k=-1) == W.ERR_INVALID_ARG  # count needed
    assert call(Wt=MISALIGNED) == W.ERR_INVALID_ARG
    assert call(y=None) == W.ERR_INVALID_ARG
    assert call(ws_bytes=need - 1) == W.ERR_WORKSPACE
    assert call(batch=0) == W.ERR_INVALID_ARG


def test_ffn_rejects_bad_arguments():
    L = W.lib
    f = W._FfnT(1 << 20, 1 << 20, 1 << 20, W.BF16, 1 << 20, 1 << 20, 1 << 20, 4096, 11008)
    need = W.workspace_size(W.OP_FFN_SWIGLU, 4096, 11008, 0, 1)

    def call(fs=f, mode=W.GATE_TOPK, kg=2048, ku=2048, kd=5504, s=0.08, ws_bytes=need, x=FAKE):
        return L.sparse_ffn_swiglu(ctypes.byref(fs) if fs is not None else None, x, W.BF16, 1, mode, kg, ku, kd, s,
                                   FAKE, FAKE, ws_bytes, None, None)

    assert call(fs=None) == W.ERR_INVALID_ARG
    assert call(kg=4097) == W.ERR_INVALID_ARG
    assert call(kd=11009) == W.ERR_INVALID_ARG
    assert call(mode=7) == W.ERR_INVALID_ARG
    assert call(mode=W.GATE_STAT, s=1.5) == W.ERR_INVALID_ARG
    assert call(ws_bytes=need - 1) == W.ERR_WORKSPACE
    assert call(x=None) == W.ERR_INVALID_ARG
    bad = W._FfnT(1 << 20, 1 << 20, 1 << 20, W.BF16, 1 << 20, 1 << 20, 1 << 20, 4096, 11000 + 4)
    assert call(fs=bad) == W.ERR_INVALID_ARG
    nodt = W._FfnT(1 << 20, 1 << 20, 1 << 20, 3, 1 << 20, 1 << 20, 1 << 20, 4096, 11008)
    assert call(fs=nodt) == W.ERR_UNSUPPORTED_DTYPE


def test_pack_and_norms_reject_bad_arguments():
    L = W.lib
    assert L.wina_pack_in_major(FAKE, W.BF16, 0, 4, FAKE, None) == W.ERR_INVALID_ARG
    assert L.wina_pack_in_major(FAKE, W.BF16, 4, 4, FAKE, None) == W.ERR_INVALID_ARG  # W and Wt overlap
    assert L.wina_pack_in_major(FAKE, 4, 4, 4, FAKE, None) == W.ERR_UNSUPPORTED_DTYPE
    assert L.wina_col_norms(FAKE, W.F32, 4, 4, 9, FAKE, None) == W.ERR_INVALID_ARG
    assert L.wina_col_norms(None, W.F32, 4, 4, 0, FAKE, None) == W.ERR_INVALID_ARG
