"""Seeded generators for the synthetic workloads.

Every array is drawn with numpy's PCG64 (``numpy.random.default_rng``). A workload's
draws happen in a fixed order from one generator, so a (workload, seed) pair always
gives the same bytes. No draw here depends on the method being tested.

Weight recipe (all workloads): for a weight W of shape [out][in], draw one scale per
input column, ``col_scale[j] ~ LogNormal(0, 0.5)`` (underlying normal: mean 0, std 0.5),
then ``W[i][j] = N(0, 1) * std * col_scale[j]``, computed in float32 and stored either
as float32 or rounded to bfloat16 (round-to-nearest-even). bf16 tensors are handed
out as their uint16 bit patterns.
"""

from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------------
# storage-format casts (not part of the method)
# ----------------------------------------------------------------------------------


def bf16_bits_from_f32(a) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits.

    The generators never produce NaN or values near the float32 overflow limit, so the
    plain bias-and-truncate rounding is exact round-to-nearest-even here.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def f32_from_bf16_bits(bits) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------------
# sizes that belong to the workload definitions
# ----------------------------------------------------------------------------------


def keep_count(p: float, n: int) -> int:
    """Kept channels K for a dropped fraction p: K = round((1 - p) * n), halves up.

    Sparsity in the WINA results is the dropped share (25%-65% sparsity); none of the
    workloads lands on an exact half, so the rounding rule never decides a tie here.
    """
    return int(math.floor((1.0 - p) * n + 0.5))


def spark_keep_count(s: float, n: int) -> int:
    """Exact top-k size used to compare against the Spark gate: k = round(s * n)."""
    return int(math.floor(s * n + 0.5))


def make_weight(rng: np.random.Generator, m: int, n: int, std: float, dtype: str) -> np.ndarray:
    """One [m][n] (out x in) weight in the recipe of the module docstring.

    dtype 'f32' returns float32 values, 'bf16' returns uint16 bf16 bits.
    """
    col_scale = rng.lognormal(mean=0.0, sigma=0.5, size=n)
    w = rng.standard_normal(size=(m, n), dtype=np.float32)
    w *= (std * col_scale).astype(np.float32)[None, :]
    if dtype == "f32":
        return w
    if dtype == "bf16":
        return bf16_bits_from_f32(w)
    raise ValueError(f"unknown dtype {dtype!r}")


# ----------------------------------------------------------------------------------
# the five workloads
# ----------------------------------------------------------------------------------


def make_linear_512x256_f32(seed: int = 0) -> dict:
    """Single fp32 linear layer: W 512x256 (out x in), N(0,1) x column log-normal(0,0.5)
    scale; x = 256 i.i.d. Laplace(0,1) in fp32; keep K = 128 (50%); batch 1."""
    rng = np.random.default_rng(seed)
    W = make_weight(rng, 512, 256, 1.0, "f32")
    x = rng.laplace(0.0, 1.0, size=(1, 256)).astype(np.float32)
    return dict(name="linear_512x256_f32", W=W, x=x, k=128, m=512, n=256, wdtype="f32", xdtype="f32")


def make_llama7b_ffn(seed: int = 1, batch: int = 1, p: float = 0.5, layer: int = 0) -> dict:
    """Llama-7B-shaped SwiGLU FFN decode: gate/up 4096->11008, down 11008->4096, bf16
    weights with std 0.02; hidden state x of Laplace(0,1) over 4096, stored as bf16.

    Draw order: W_gate, W_up, W_down, then x[batch][4096]. ``layer`` selects an
    independent stream (distinct weight copies for multi-layer timing).
    """
    d, ffn = 4096, 11008
    rng = np.random.default_rng((seed, layer))
    Wg = make_weight(rng, ffn, d, 0.02, "bf16")
    Wu = make_weight(rng, ffn, d, 0.02, "bf16")
    Wd = make_weight(rng, d, ffn, 0.02, "bf16")
    x = bf16_bits_from_f32(rng.laplace(0.0, 1.0, size=(batch, d)).astype(np.float32))
    return dict(
        name="llama7b_ffn_4096x11008_bf16", d=d, ffn=ffn, Wg=Wg, Wu=Wu, Wd=Wd, x=x, p=p,
        k_gate=keep_count(p, d), k_up=keep_count(p, d), k_down=keep_count(p, ffn),
    )


LLAMA3_8B_PROJ = (
    # name, in, out
    ("q", 4096, 4096),
    ("k", 4096, 1024),
    ("v", 4096, 1024),
    ("o", 4096, 4096),
    ("gate", 4096, 14336),
    ("up", 4096, 14336),
    ("down", 14336, 4096),
)


def make_llama3_8b_layer(seed: int = 2, batch: int = 16, only: tuple | None = None) -> dict:
    """Llama-3-8B-shaped decoder layer, bf16 (std 0.02): Q 4096->4096, K/V 4096->1024,
    O 4096->4096, gate/up 4096->14336, down 14336->4096.

    Draw order: seven per-projection dropped fractions p ~ U(0.4, 0.7) (in the order of
    ``LLAMA3_8B_PROJ``), the seven weights in that order, then x[batch][4096]
    (Laplace(0,1); input of Q, K, V, gate and up) and o_in[batch][4096] (Laplace(0,1);
    the O projection's input, since no attention core is in scope). The down
    projection's input is h = silu(gate) * up, computed by whoever runs the layer.
    ``only`` limits which weights are materialised (the others are still drawn, so the
    streams stay aligned, but dropped at once).
    """
    rng = np.random.default_rng(seed)
    ps = rng.uniform(0.4, 0.7, size=len(LLAMA3_8B_PROJ))
    out = dict(name="llama3_8b_layer_bf16", p={}, k={}, W={}, shape={})
    for (name, n_in, n_out), p in zip(LLAMA3_8B_PROJ, ps):
        w = make_weight(rng, n_out, n_in, 0.02, "bf16")
        out["p"][name] = float(p)
        out["k"][name] = keep_count(float(p), n_in)
        out["shape"][name] = (n_out, n_in)
        if only is None or name in only:
            out["W"][name] = w
        del w
    out["x"] = bf16_bits_from_f32(rng.laplace(0.0, 1.0, size=(batch, 4096)).astype(np.float32))
    out["o_in"] = bf16_bits_from_f32(rng.laplace(0.0, 1.0, size=(batch, 4096)).astype(np.float32))
    return out


def make_gemma2_2b_spark(seed: int = 3, batch: int = 64, s: float = 0.08, weights: bool = True) -> dict:
    """Gemma-2-2B-shaped FFN for the Spark statistical gate: d = 2304, ffn = 9216, bf16
    weights (std 0.02); keep fraction s = 0.08.

    Draw order: W_gate [9216][2304], W_up, W_down [2304][9216] (skipped when
    ``weights`` is False), then per token b: mu_b ~ U(-0.1, 0.1), sigma_b ~ U(0.5, 2),
    x_b ~ N(mu_b, sigma_b^2) over 2304; then again per token an independent
    mu'_b, sigma'_b and v_b ~ N(mu'_b, sigma'_b^2) over 9216 (a stand-alone input of
    the length of the down projection). x and v are float32; ``x_bf16`` is x rounded
    to bf16 for the FFN call.
    """
    d, ffn = 2304, 9216
    rng = np.random.default_rng(seed)
    out = dict(name="gemma2_2b_ffn_spark_2304x9216_bf16", d=d, ffn=ffn, s=s)
    if weights:
        out["Wg"] = make_weight(rng, ffn, d, 0.02, "bf16")
        out["Wu"] = make_weight(rng, ffn, d, 0.02, "bf16")
        out["Wd"] = make_weight(rng, d, ffn, 0.02, "bf16")
    mu = rng.uniform(-0.1, 0.1, size=batch)
    sig = rng.uniform(0.5, 2.0, size=batch)
    x = (mu[:, None] + sig[:, None] * rng.standard_normal(size=(batch, d))).astype(np.float32)
    mu2 = rng.uniform(-0.1, 0.1, size=batch)
    sig2 = rng.uniform(0.5, 2.0, size=batch)
    v = (mu2[:, None] + sig2[:, None] * rng.standard_normal(size=(batch, ffn))).astype(np.float32)
    out.update(x=x, x_bf16=bf16_bits_from_f32(x), v=v, mu=mu, sigma=sig, mu_v=mu2, sigma_v=sig2,
               k_d=spark_keep_count(s, d), k_ffn=spark_keep_count(s, ffn))
    return out


def make_ultrasparse_down(seed: int = 4, batch: int = 256, nnz_frac: float = 0.01) -> dict:
    """Ultra-sparse (L1-regularised, ReLU-style) down projection 14336 -> 4096, bf16
    weights (std 0.02); per token round(0.01 * 14336) = 143 nonzero inputs at distinct
    uniformly random positions with Exponential(1) magnitudes, stored as bf16; 256 tokens.

    Draw order: W [4096][14336], then per token: the positions (without replacement),
    then the magnitudes.
    """
    n, m = 14336, 4096
    nnz = int(math.floor(nnz_frac * n + 0.5))
    rng = np.random.default_rng(seed)
    W = make_weight(rng, m, n, 0.02, "bf16")
    x = np.zeros((batch, n), dtype=np.float32)
    for b in range(batch):
        pos = rng.choice(n, size=nnz, replace=False)
        x[b, pos] = rng.exponential(1.0, size=nnz).astype(np.float32)
    return dict(name="ultrasparse_down_14336x4096_b256", W=W, x=bf16_bits_from_f32(x), n=n, m=m, nnz=nnz)


def make_ds_decode(seed: int = 5, batch: int = 1, hq: int = 32, hkv: int = 32, seq=4096, dh: int = 128,
                   n_outlier: int = 16, outlier_scale: float = 4.0, tmax: int | None = None) -> dict:
    """Double Sparsity decode workload (Llama-2-7B attention shapes by default: 32 query
    and 32 key/value heads of 128 channels, 4096 cached tokens, bf16 caches).

    Draw order: per key/value head g, a set O_g of ``n_outlier`` distinct channels
    (uniform, without replacement); then K [B][Hkv][Tmax][dh] ~ N(0, 1) with the channels
    of O_g multiplied by ``outlier_scale``; then V ~ N(0, 1); then q [B][Hq][dh] ~ N(0, 1)
    with the channels of its key/value head's O_g multiplied by ``outlier_scale`` (so that
    a few channels carry most of q . K, the structure the method relies on). ``seq`` is
    one length for every sequence or a list of B lengths; cache slots past a sequence's
    length hold draws too (they must not be read). Caches and q are bf16 bit patterns.
    """
    rng = np.random.default_rng(seed)
    seq_len = np.array([seq] * batch if np.isscalar(seq) else list(seq), dtype=np.int32)
    T = int(tmax if tmax is not None else seq_len.max())
    outl = np.stack([np.sort(rng.choice(dh, size=n_outlier, replace=False)) for _ in range(hkv)]).astype(np.int32)
    colscale = np.ones((hkv, dh), dtype=np.float32)
    for g in range(hkv):
        colscale[g, outl[g]] = outlier_scale
    K = (rng.standard_normal((batch, hkv, T, dh), dtype=np.float32) * colscale[None, :, None, :]).astype(np.float32)
    V = rng.standard_normal((batch, hkv, T, dh), dtype=np.float32)
    grp = hq // hkv
    qs = colscale[np.arange(hq) // grp]
    q = (rng.standard_normal((batch, hq, dh), dtype=np.float32) * qs[None]).astype(np.float32)
    return dict(name=f"ds_decode_b{batch}_h{hq}x{hkv}_t{T}_d{dh}", K=bf16_bits_from_f32(K), V=bf16_bits_from_f32(V),
                q=bf16_bits_from_f32(q), seq_len=seq_len, outliers=outl, B=batch, Hq=hq, Hkv=hkv, Tmax=T, dh=dh)


WORKLOADS = {
    "linear_512x256_f32": make_linear_512x256_f32,
    "llama7b_ffn_4096x11008_bf16": make_llama7b_ffn,
    "llama3_8b_layer_bf16": make_llama3_8b_layer,
    "gemma2_2b_ffn_spark_2304x9216_bf16": make_gemma2_2b_spark,
    "ultrasparse_down_14336x4096_b256": make_ultrasparse_down,
    "ds_decode_llama2_7b_t4096": make_ds_decode,
}
