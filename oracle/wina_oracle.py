"""Plain, slow CPU oracle (numpy, float64) for the weight-informed activation-sparse
linear layer and the SwiGLU FFN built from it.

TEST INFRASTRUCTURE ONLY: imported solely by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference leg. The CUDA path never routes through it.
It shares no code, table or helper with the CUDA library.

Sources (web pages on training-free activation sparsity; cited by title and section):

* [WINA] "WINA: Weight Informed Neuron Activation" article (lsdiaocha.cn, 2025-05-29),
  section 一 (weight-aware activation: the gate), section 二 (theoretical basis: the
  single-layer error bound for column-orthogonal W), section 五 (the SVD transform,
  W' = WV with W'^T W' = Sigma^2), section 三 (sparsity levels 25%-65%).
* [Spark] "Spark Transformer: 高效稀疏化大语言模型架构设计" (intelliparadigm.com),
  section 2.2 (statistical top-k operator), section 3.1 (the VMM / SVMM primitives),
  section 2.1 (FFN as a key-value lookup).
* [WAS] "哈工大EMNLP 2025论文开源: 贝叶斯优化驱动的LLM激活稀疏加速框架" (zingnex.cn),
  section "WAS框架的核心创新" (weight-aware sparsity applied per component:
  Q, K, V, O, gate, up, down).

Readings taken where the pages are silent:

* ties in the top-K gate go to the lower channel index; the kept set is returned as an
  ascending index list;
* the gate score is computed in float32: one IEEE multiply x_i * c_i rounded to
  nearest-even, then the absolute value; c is stored as float32;
* c_j is accumulated in float64 and rounded once to float32;
* the Spark variance divides by n (population form), its comparison is strict (v > t)
  and it thresholds the signed input vector; Phi^-1 is the standard normal quantile;
* between the FFN's projections h is held in float32; the down gate scores that
  float32 h.
"""

from __future__ import annotations

import math
from statistics import NormalDist

import numpy as np

__all__ = [
    "widen_bf16",
    "col_norms",
    "gate_scores",
    "select_topk",
    "wina_select",
    "teal_select",
    "svd_transform",
    "sparse_matvec",
    "sparse_matvec_rows",
    "dense_matvec",
    "silu",
    "ffn_swiglu",
    "spark_threshold",
    "spark_ffn",
    "exact_topk_signed",
    "overlap",
    "output_error",
    "union_indices",
]


def widen_bf16(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64 values (exact: bf16 is the top half of binary32)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------------------
# the gate ([WINA] section 一)
# --------------------------------------------------------------------------------------


def col_norms(W) -> np.ndarray:
    """Column-wise l2 norms of W ([WINA] section 一: c holds the l2 norm of each column
    of W; section 二 writes the same quantity as ||W_{.,j}||_2).

    W is [out][in] (the matrix that multiplies x). c_j = sqrt(sum_i W_ij^2), summed in
    float64, square root in float64, then rounded once to float32.
    """
    W = np.asarray(W, dtype=np.float64)
    sq = W * W
    return np.sqrt(sq.sum(axis=0)).astype(np.float32)


def gate_scores(x, c=None) -> np.ndarray:
    """Per-channel gate score |x_i * c_i| ([WINA] section 一: the score vector is the
    absolute value of the Hadamard product x (.) c).

    Computed in float32: one IEEE multiply, then abs. ``c=None`` gives the
    magnitude-only gate |x_i| of TEAL/CATS, the comparator in [WINA] section 二.
    """
    x32 = np.asarray(x, dtype=np.float32)
    if c is None:
        return np.abs(x32)
    return np.abs(x32 * np.asarray(c, dtype=np.float32))


def select_topk(score, k: int) -> np.ndarray:
    """Binary gate m_i = 1 iff score_i is among the K largest ([WINA] section 一).

    Explicit stable sort on the key (-score_i, i): larger score first, equal scores in
    ascending index order, so ties at the K-th value keep the lower index. Returns the
    kept indices in ascending order (int32).
    """
    s = np.asarray(score, dtype=np.float32).astype(np.float64)
    n = s.shape[0]
    if not 0 <= k <= n:
        raise ValueError(f"k={k} outside [0, {n}]")
    order = np.lexsort((np.arange(n), -s))  # primary key -score, secondary key index
    return np.sort(order[:k]).astype(np.int32)


def wina_select(x, c, k: int) -> np.ndarray:
    """WINA gate: ascending indices of the top-K of |x (.) c| ([WINA] section 一)."""
    return select_topk(gate_scores(x, c), k)


def teal_select(x, k: int) -> np.ndarray:
    """TEAL/CATS gate: top-K of |x| alone ([WINA] section 二, the comparator)."""
    return select_topk(gate_scores(x, None), k)


# --------------------------------------------------------------------------------------
# the sparse product ([Spark] section 3.1, SVMM)
# --------------------------------------------------------------------------------------


def sparse_matvec(W, idx, xs) -> np.ndarray:
    """y = sum over the active channels j of xs_j * W[:, j] ([Spark] section 3.1: the
    sparse-vector x matrix loop that visits only the active indices; [WINA] section 一:
    only the selected neurons take part).

    W is [out][in]; idx are input-channel indices, xs their input values. float64.
    """
    W = np.asarray(W, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    xs = np.asarray(xs, dtype=np.float64)
    if idx.size == 0:
        return np.zeros(W.shape[0], dtype=np.float64)
    return W[:, idx] @ xs


def sparse_matvec_rows(W_rows, idx, xs) -> np.ndarray:
    """Selected outputs of the sparse product: W_rows are some rows of W ([r][in]), the
    result is those r outputs of ``sparse_matvec``. Used to check sampled outputs of
    full-size layers one by one."""
    return sparse_matvec(W_rows, idx, xs)


def dense_matvec(W, x) -> np.ndarray:
    """y = W x in float64 (the unsparsified layer)."""
    return np.asarray(W, dtype=np.float64) @ np.asarray(x, dtype=np.float64)


def union_indices(idx_lists) -> np.ndarray:
    """Union of several tokens' kept index sets, ascending (int32)."""
    if len(idx_lists) == 0:
        return np.zeros(0, dtype=np.int32)
    return np.unique(np.concatenate([np.asarray(i, dtype=np.int64) for i in idx_lists])).astype(np.int32)


# --------------------------------------------------------------------------------------
# SwiGLU FFN with the gate on every projection ([WAS] core innovations; [WINA] 一, 五)
# --------------------------------------------------------------------------------------


def silu(g):
    """silu(g) = g / (1 + exp(-g)), float64."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def ffn_swiglu(Wg, Wu, Wd, cg, cu, cd, x, kg: int, ku: int, kd: int, mode: str = "topk", s: float = 0.08) -> dict:
    """One token through a SwiGLU FFN whose three projections are each gated.

    The gate is applied to every projection's own input, with that projection's own
    column norms ([WAS]: weight-aware sparsity per component, gate/up/down among them;
    [WINA] section 一: K may differ per layer). Steps:

      S_g = gate(x, c_gate, K_g);  g = W_gate[:, S_g] x[S_g]
      S_u = gate(x, c_up,   K_u);  u = W_up[:, S_u]   x[S_u]
      h   = silu(g) * u                       (float64, then held as float32)
      S_d = gate(h, c_down, K_d);  y = W_down[:, S_d] h[S_d]

    ``mode='topk'`` uses the WINA top-K gate; ``mode='stat'`` uses the Spark threshold
    on each projection's signed input ([Spark] section 2.2) and ignores the c's and K's.
    Weights are [out][in] float64-convertible arrays.
    """
    x = np.asarray(x)
    if mode == "topk":
        ig = wina_select(x, cg, kg)
        iu = wina_select(x, cu, ku)
    elif mode == "stat":
        ig = spark_threshold(x, s)["idx"]
        iu = ig
    else:
        raise ValueError(mode)
    x64 = np.asarray(x, dtype=np.float64)
    g = sparse_matvec(Wg, ig, x64[ig])
    u = sparse_matvec(Wu, iu, x64[iu])
    h = silu(g) * u
    h32 = h.astype(np.float32)
    if mode == "topk":
        idn = wina_select(h32, cd, kd)
    else:
        idn = spark_threshold(h32, s)["idx"]
    y = sparse_matvec(Wd, idn, h[idn])
    return dict(idx_gate=ig, idx_up=iu, g=g, u=u, h=h, h32=h32, idx_down=idn, y=y)


# --------------------------------------------------------------------------------------
# Spark statistical top-k ([Spark] section 2.2)
# --------------------------------------------------------------------------------------


def spark_threshold(v, s: float) -> dict:
    """Statistical top-k of [Spark] section 2.2: model the entries of v as Gaussian,
    estimate mu = mean(v) and sigma^2 = mean((v - mu)^2) (divisor n), set
    t = mu + sigma * Phi^-1(1 - s) for keep fraction s, and keep {i : v_i > t}.

    float64 throughout; Phi^-1 from the standard library's NormalDist.
    """
    if not 0.0 < s < 1.0:
        raise ValueError("keep fraction s must lie in (0, 1)")
    v = np.asarray(v, dtype=np.float64)
    mu = float(v.mean())
    var = float(((v - mu) ** 2).mean())
    sigma = math.sqrt(var)
    z = NormalDist().inv_cdf(1.0 - s)
    t = mu + sigma * z
    idx = np.nonzero(v > t)[0].astype(np.int32)
    return dict(mu=mu, var=var, sigma=sigma, z=z, t=t, idx=idx)


def spark_ffn(Wg, Wu, Wd, x, s: float) -> dict:
    """The Spark FFN as a key-value lookup ([Spark] section 2.1: y = sum_i f(q . k_i) v_i;
    compute the dot products of the query with every key, keep the neurons the
    statistical top-k selects, activate only those), for a SwiGLU FFN:

      g   = W_gate x                         (every neuron's pre-activation: the scores)
      S   = spark_threshold(g, s)             ([Spark] section 2.2, on the signed float32 g)
      h_i = silu(g_i) * (W_up[i] . x)   for i in S
      y   = W_down[:, S] h[S]

    Weights are [out][in]: W_gate, W_up [ffn][d], W_down [d][ffn]. float64 arithmetic; g
    is held in float32 for the selection (as the scores of the gate are).
    """
    Wg = np.asarray(Wg, dtype=np.float64)
    Wu = np.asarray(Wu, dtype=np.float64)
    Wd = np.asarray(Wd, dtype=np.float64)
    x64 = np.asarray(x, dtype=np.float64)
    g = Wg @ x64
    g32 = g.astype(np.float32)
    S = spark_threshold(g32, s)["idx"]
    u = Wu[S] @ x64
    h = silu(g[S]) * u
    y = Wd[:, S] @ h if S.size else np.zeros(Wd.shape[0])
    return dict(g=g, g32=g32, idx=S, u=u, h=h, y=y)


def exact_topk_signed(v, k: int) -> np.ndarray:
    """Exact top-k of the signed values (largest first, ties to the lower index),
    ascending indices: the set the statistical operator approximates ([Spark] 2.2)."""
    return select_topk(np.asarray(v, dtype=np.float32), k)


def overlap(S, T) -> dict:
    """|S & T| / |T| and the Jaccard index |S & T| / |S | T| of two index sets."""
    S = set(int(i) for i in S)
    T = set(int(i) for i in T)
    inter = len(S & T)
    uni = len(S | T)
    return dict(inter=inter, recall=(inter / len(T)) if T else 1.0, jaccard=(inter / uni) if uni else 1.0)


# --------------------------------------------------------------------------------------
# the approximation error the theorem speaks of ([WINA] section 二)
# --------------------------------------------------------------------------------------


def svd_transform(W):
    """The column-orthogonalising transform of [WINA] section 五: with the thin SVD
    W = U diag(s) V^T, W' = W V = U diag(s) has orthogonal columns (W'^T W' = diag(s^2),
    column norms s), and W' (V^T x) = W x, so the gate can run on W' and x' = V^T x without
    changing the layer's output. Returns (W', V) in float64. Offline; not on the path."""
    W64 = np.asarray(W, dtype=np.float64)
    _, _, vt = np.linalg.svd(W64, full_matrices=False)
    V = vt.T
    return W64 @ V, V


def output_error(W, x, idx) -> float:
    """Squared output error of a gate: ||W x - W (m (.) x)||_2^2 with m the indicator of
    the kept set ([WINA] section 二 bounds the expectation of this error)."""
    x64 = np.asarray(x, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    full = dense_matvec(W, x64)
    kept = sparse_matvec(W, idx, x64[idx])
    d = full - kept
    return float(d @ d)
