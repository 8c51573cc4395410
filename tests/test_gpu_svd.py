"""The column-orthogonalising transform of the WINA article (section 五) on the GPU path.

W' = W V and x' = V^T x (V from the SVD of W, computed on the CPU by the oracle) leave the
layer's output unchanged, W' x' = W x, and give W' orthogonal columns, for which the WINA
gate keeps exactly the error-minimising set. The transformed weight and input go through
the CUDA path like any other (wina_col_norms -> wina_select_topk -> sparse_matvec) and are
compared with the oracle: identical kept sets (same float32 scores), the product within
the stated bound, and, at small sizes, the GPU's kept set equal to the brute-force
minimiser of ||W' x' - W' (m * x')||^2 over all K-subsets.
"""

from __future__ import annotations

import itertools

import numpy as np
import pytest

import oracle as O
import free_activation_sparse_b200 as W
from tests.gpu_util import dev_f32, host, rel_l2

pytestmark = pytest.mark.gpu


def _transformed(rng, m, n):
    # correlated columns with unequal scales, so that the transform matters
    Wm = (rng.standard_normal((m, n)) @ (np.eye(n) + 0.3 * rng.standard_normal((n, n)))) * rng.lognormal(0, 0.5, n)
    Wp, V = O.svd_transform(Wm)
    return Wm, Wp.astype(np.float32), V


@pytest.mark.parametrize("m,n,k", [(512, 256, 128), (1024, 384, 100)])
def test_svd_transform_on_gpu_path(m, n, k):
    rng = np.random.default_rng(m + n)
    Wm, Wp32, V = _transformed(rng, m, n)
    x = rng.laplace(size=n)
    xp = (V.T @ x).astype(np.float32)
    c_gpu = host(W.col_norms(dev_f32(Wp32)))
    c_ref = O.col_norms(Wp32)
    assert np.array_equal(c_gpu, c_ref)
    idx_d, xs_d = W.select_topk(dev_f32(xp), dev_f32(c_gpu), k)
    idx = host(idx_d)[0]
    assert np.array_equal(idx, O.wina_select(xp, c_ref, k))
    y = host(W.sparse_matvec(W.pack_in_major(dev_f32(Wp32)), idx_d, xs_d))[0]
    want = O.sparse_matvec(Wp32.astype(np.float64), idx, xp[idx].astype(np.float64))
    assert rel_l2(y, want) <= 1e-5
    # with every channel kept the transformed layer reproduces the original output
    idx_all, xs_all = W.select_topk(dev_f32(xp), dev_f32(c_gpu), n)
    y_all = host(W.sparse_matvec(W.pack_in_major(dev_f32(Wp32)), idx_all, xs_all))[0]
    assert rel_l2(y_all, O.dense_matvec(Wm, x)) <= 1e-4


@pytest.mark.parametrize("seed", range(4))
def test_gpu_set_is_the_error_minimiser_after_the_transform(seed):
    rng = np.random.default_rng(100 + seed)
    m, n = 20, 10
    _, Wp32, V = _transformed(rng, m, n)
    Wp = Wp32.astype(np.float64)
    xp = (V.T @ rng.laplace(size=n)).astype(np.float32)
    c = host(W.col_norms(dev_f32(Wp32)))
    for k in (1, 3, 5, 8):
        got = host(W.select_topk(dev_f32(xp), dev_f32(c), k)[0])[0]
        errs = {S: O.output_error(Wp, xp, np.array(S)) for S in itertools.combinations(range(n), k)}
        best = min(errs.values())
        # the GPU's set attains the minimum (other sets may tie only within rounding)
        assert errs[tuple(int(i) for i in got)] <= best * (1 + 1e-6) + 1e-12
