"""Weight-informed activation-sparse linear layer for LLM decode on B200 (sm_100a).

A thin ctypes binding of ``libwina.so`` (the C ABI in ``include/wina.h``). Every step
of the computation runs in the library's CUDA kernels; this module only checks tensor
dtypes/devices, allocates outputs and workspaces through PyTorch, passes raw device
pointers and the current CUDA stream, and turns status codes into exceptions.
Importing it fails if the library has not been built
(``python free_activation_sparse_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

__all__ = [
    "WinaError", "lib", "LIB_PATH", "F32", "BF16", "GATE_TOPK", "GATE_STAT", "GATE_DENSE",
    "abi_version", "normal_quantile", "workspace_size", "Workspace", "FfnWeights",
    "pack_in_major", "col_norms", "select_topk", "stat_topk_threshold", "sparse_matvec",
    "sparse_ffn_swiglu", "ffn_ws_view", "ffn_prepare", "declared_symbols", "sparse_matvec_noalloc",
    "dense_matvec", "dense_ffn_swiglu", "spark_ffn", "ds_channel_absmean", "ds_calibrate_channels",
    "ds_label_build", "ds_decode_attention",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwina.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "wina.h")

# enums of wina.h
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_DTYPE, ERR_WORKSPACE, ERR_CAPACITY, ERR_CUDA, ERR_TIMEOUT = range(7)
F32, BF16 = 0, 1
LAYOUT_OUT_IN, LAYOUT_IN_MAJOR = 0, 1
GATE_TOPK, GATE_STAT, GATE_DENSE = 0, 1, 2
OP_SELECT_TOPK, OP_STAT_THRESHOLD, OP_SPARSE_MATVEC, OP_FFN_SWIGLU, OP_SPARK_FFN, OP_DENSE_FFN = 0, 1, 2, 3, 4, 5


class WinaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {lib.wina_status_string(code).decode()} (status {code})")


class _FfnT(ctypes.Structure):
    _fields_ = [
        ("wt_gate", ctypes.c_void_p), ("wt_up", ctypes.c_void_p), ("wt_down", ctypes.c_void_p),
        ("wdt", ctypes.c_int), ("c_gate", ctypes.c_void_p), ("c_up", ctypes.c_void_p),
        ("c_down", ctypes.c_void_p), ("d", ctypes.c_int64), ("ffn", ctypes.c_int64),
    ]


class _FfnView(ctypes.Structure):
    _fields_ = [("h", ctypes.c_size_t), ("keep_gate", ctypes.c_size_t), ("keep_up", ctypes.c_size_t),
                ("keep_down", ctypes.c_size_t), ("stamps", ctypes.c_size_t), ("cta_t", ctypes.c_size_t)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python free_activation_sparse_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I32, D, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_size_t
    E = ctypes.c_int
    sig = {
        "wina_abi_version": (I32, []),
        "wina_set_wait_limit_ns": (None, [ctypes.c_uint64]),
        "wina_status_string": (ctypes.c_char_p, [E]),
        "wina_normal_quantile": (D, [D]),
        "wina_workspace_size": (SZ, [E, I64, I64, I64, I64]),
        "wina_ffn_ws_view": (E, [I64, I64, I64, ctypes.POINTER(_FfnView)]),
        "wina_pack_in_major": (E, [P, E, I64, I64, P, P]),
        "wina_col_norms": (E, [P, E, I64, I64, E, P, P]),
        "wina_select_topk": (E, [P, E, P, I64, I64, I64, P, P, P, P]),
        "stat_topk_threshold": (E, [P, E, I64, D, I64, P, P, P, P, I64, P, P]),
        "sparse_matvec": (E, [P, E, I64, I64, P, P, I64, P, I64, I64, P, P, SZ, P, P]),
        "sparse_matvec_noalloc": (E, [P, E, I64, I64, P, P, I64, P, I64, I64, P, P, P]),
        "sparse_ffn_swiglu": (E, [ctypes.POINTER(_FfnT), P, E, I64, E, I64, I64, I64, D, P, P, SZ, P, P]),
        "wina_dense_matvec": (E, [P, E, I64, I64, P, E, P, P, P]),
        "spark_ffn_swiglu": (E, [P, P, P, E, I64, I64, P, E, D, P, P, P, P, P, SZ, P, P]),
        "wina_dense_ffn_swiglu": (E, [P, P, P, E, I64, I64, P, E, P, P, SZ, P, P]),
        "ds_channel_absmean": (E, [P, E, I64, I64, I64, I64, P, P, P]),
        "ds_label_build": (E, [P, E, I64, I64, I64, I64, P, P, I64, I64, I64, P, P]),
        "ds_decode_smem_bytes": (SZ, [I64, I64, I64]),
        "ds_decode_attention": (E, [P, E, P, P, P, E, P, I64, I64, I64, I64, I64, I64, P, I64, ctypes.c_float, P, P, P,
                                    P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def declared_symbols() -> list[str]:
    """Function names declared in include/wina.h (parsed from the header text)."""
    import re
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)) - {"defined"})


# ------------------------------------------------------------------------------------
# marshalling helpers (no arithmetic of the method here)
# ------------------------------------------------------------------------------------


def _torch():
    import torch
    return torch


def _dt(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _cuda(t, name):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check(code: int, where: str):
    if code != OK:
        raise WinaError(code, where)


def abi_version() -> int:
    return int(lib.wina_abi_version())


def normal_quantile(p: float) -> float:
    """Phi^-1(p), computed by the library's host code."""
    return float(lib.wina_normal_quantile(float(p)))


def workspace_size(op: int, n: int, m: int, k: int, batch: int) -> int:
    return int(lib.wina_workspace_size(int(op), int(n), int(m), int(k), int(batch)))


class Workspace:
    """A zero-filled device scratch buffer for one op and size (reusable across calls
    of that op on one stream)."""

    def __init__(self, op: int, n: int, m: int, k: int, batch: int, device=None):
        torch = _torch()
        nbytes = max(workspace_size(op, n, m, k, batch), 256)
        self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")
        self.nbytes = nbytes

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


# ------------------------------------------------------------------------------------
# public calls
# ------------------------------------------------------------------------------------


def pack_in_major(W):
    """W[m][n] -> Wt[n][m] (input-channel-major), same dtype."""
    torch = _torch()
    _cuda(W, "W")
    m, n = W.shape
    Wt = torch.empty((n, m), dtype=W.dtype, device=W.device)
    _check(lib.wina_pack_in_major(_ptr(W), _dt(W), m, n, _ptr(Wt), _stream()), "wina_pack_in_major")
    return Wt


def col_norms(W, layout: str = "out_in"):
    """float32 column norms c[n] of W[m][n] ('out_in') or of the packed Wt[n][m] ('in_major')."""
    torch = _torch()
    _cuda(W, "W")
    if layout == "out_in":
        m, n = W.shape
        lay = LAYOUT_OUT_IN
    elif layout == "in_major":
        n, m = W.shape
        lay = LAYOUT_IN_MAJOR
    else:
        raise ValueError(layout)
    c = torch.empty(n, dtype=torch.float32, device=W.device)
    _check(lib.wina_col_norms(_ptr(W), _dt(W), m, n, lay, _ptr(c), _stream()), "wina_col_norms")
    return c


def select_topk(x, c, k: int, want_scores: bool = False):
    """Top-k gate per token: returns (idx int32 [B][k] ascending, xs float32 [B][k]
    [, scores float32 [B][n]])."""
    torch = _torch()
    _cuda(x, "x")
    _cuda(c, "c")
    x2 = x.reshape(1, -1) if x.dim() == 1 else x
    B, n = x2.shape
    idx = torch.empty((B, k), dtype=torch.int32, device=x.device)
    xs = torch.empty((B, k), dtype=torch.float32, device=x.device)
    sc = torch.empty((B, n), dtype=torch.float32, device=x.device) if want_scores else None
    _check(lib.wina_select_topk(_ptr(x2), _dt(x2), _ptr(c), n, k, B, _ptr(idx), _ptr(xs), _ptr(sc), _stream()),
           "wina_select_topk")
    return (idx, xs, sc) if want_scores else (idx, xs)


def stat_topk_threshold(v, s: float, cap: int | None = None, status=None):
    """Spark statistical gate per row of v: returns (idx [B][cap], xs [B][cap],
    count [B], t [B]). Entries past count are unspecified."""
    torch = _torch()
    _cuda(v, "v")
    v2 = v.reshape(1, -1) if v.dim() == 1 else v
    B, n = v2.shape
    cap = n if cap is None else int(cap)
    idx = torch.empty((B, max(cap, 1)), dtype=torch.int32, device=v.device)
    xs = torch.empty((B, max(cap, 1)), dtype=torch.float32, device=v.device)
    count = torch.empty(B, dtype=torch.int32, device=v.device)
    t = torch.empty(B, dtype=torch.float32, device=v.device)
    _check(lib.stat_topk_threshold(_ptr(v2), _dt(v2), n, float(s), B, _ptr(idx), _ptr(xs), _ptr(count), _ptr(t),
                                   cap, _ptr(status), _stream()), "stat_topk_threshold")
    return idx[:, :cap], xs[:, :cap], count, t


def sparse_matvec(Wt, idx, xs, k: int | None = None, count=None, ws: Workspace | None = None, status=None, y=None):
    """y[b] = sum_r xs[b][r] * Wt[idx[b][r]] over the first k (or count[b]) entries."""
    torch = _torch()
    for t_, nm in ((Wt, "Wt"), (idx, "idx"), (xs, "xs"), (count, "count")):
        _cuda(t_, nm)
    if idx.dtype != torch.int32 or xs.dtype != torch.float32:
        raise TypeError("idx must be int32 and xs float32")
    idx2 = idx.reshape(1, -1) if idx.dim() == 1 else idx
    xs2 = xs.reshape(1, -1) if xs.dim() == 1 else xs
    n, m = Wt.shape
    B, ld = idx2.shape
    if k is None and count is None:
        k = ld
    kk = -1 if k is None else int(k)
    if ws is None:
        ws = Workspace(OP_SPARSE_MATVEC, n, m, ld, B, device=Wt.device)
    if y is None:
        y = torch.empty((B, m), dtype=torch.float32, device=Wt.device)
    _check(lib.sparse_matvec(_ptr(Wt), _dt(Wt), n, m, _ptr(idx2), _ptr(xs2), kk, _ptr(count), ld, B, _ptr(y),
                             ws.ptr, ws.nbytes, _ptr(status), _stream()), "sparse_matvec")
    return y


def sparse_matvec_noalloc(Wt, idx, xs, k: int | None = None, count=None, status=None, y=None):
    """sparse_matvec without a workspace: the library's own fixed scratch is used (for
    callers that cannot allocate device memory; see include/wina.h for its limit and
    the rule that such calls must not overlap)."""
    torch = _torch()
    for t_, nm in ((Wt, "Wt"), (idx, "idx"), (xs, "xs"), (count, "count")):
        _cuda(t_, nm)
    if idx.dtype != torch.int32 or xs.dtype != torch.float32:
        raise TypeError("idx must be int32 and xs float32")
    idx2 = idx.reshape(1, -1) if idx.dim() == 1 else idx
    xs2 = xs.reshape(1, -1) if xs.dim() == 1 else xs
    n, m = Wt.shape
    B, ld = idx2.shape
    if k is None and count is None:
        k = ld
    kk = -1 if k is None else int(k)
    if y is None:
        y = torch.empty((B, m), dtype=torch.float32, device=Wt.device)
    _check(lib.sparse_matvec_noalloc(_ptr(Wt), _dt(Wt), n, m, _ptr(idx2), _ptr(xs2), kk, _ptr(count), ld, B,
                                     _ptr(y), _ptr(status), _stream()), "sparse_matvec_noalloc")
    return y


@dataclass
class FfnWeights:
    """Packed SwiGLU FFN: wt_gate/wt_up [d][ffn], wt_down [ffn][d] (input-major), and
    the float32 column norms of W_gate, W_up (length d) and W_down (length ffn)."""
    wt_gate: object
    wt_up: object
    wt_down: object
    c_gate: object
    c_up: object
    c_down: object

    @property
    def d(self) -> int:
        return int(self.wt_gate.shape[0])

    @property
    def ffn(self) -> int:
        return int(self.wt_gate.shape[1])

    def _struct(self) -> _FfnT:
        key = (self.wt_gate.data_ptr(), self.wt_up.data_ptr(), self.wt_down.data_ptr(), self.c_gate.data_ptr(),
               self.c_up.data_ptr(), self.c_down.data_ptr())
        cached = self.__dict__.get("_cstruct")
        if cached is None or cached[0] != key:
            st = _FfnT(key[0], key[1], key[2], _dt(self.wt_gate), key[3], key[4], key[5], self.d, self.ffn)
            self.__dict__["_cstruct"] = cached = (key, st)
        return cached[1]


def ffn_prepare(W_gate, W_up, W_down) -> FfnWeights:
    """Offline preparation of one FFN from W_gate, W_up [ffn][d] and W_down [d][ffn]
    (output-major, as multiplied by x): pack input-major and take column norms."""
    return FfnWeights(pack_in_major(W_gate), pack_in_major(W_up), pack_in_major(W_down),
                      col_norms(W_gate), col_norms(W_up), col_norms(W_down))


def sparse_ffn_swiglu(f: FfnWeights, x, mode: int = GATE_TOPK, k_gate: int = 0, k_up: int = 0, k_down: int = 0,
                      s: float = 0.08, ws: Workspace | None = None, status=None, y=None):
    """Gated SwiGLU FFN for x [B][d]: returns y float32 [B][d]."""
    torch = _torch()
    _cuda(x, "x")
    x2 = x.reshape(1, -1) if x.dim() == 1 else x
    B = x2.shape[0]
    if ws is None:
        ws = Workspace(OP_FFN_SWIGLU, f.d, f.ffn, 0, B, device=x.device)
    if y is None:
        y = torch.empty((B, f.d), dtype=torch.float32, device=x.device)
    _check(lib.sparse_ffn_swiglu(ctypes.byref(f._struct()), _ptr(x2), _dt(x2), B, int(mode), int(k_gate), int(k_up),
                                 int(k_down), float(s), _ptr(y), ws.ptr, ws.nbytes, _ptr(status), _stream()),
           "sparse_ffn_swiglu")
    return y


def dense_matvec(W, x, y=None, xbuf=None):
    """The dense comparator y = W x on the output-major W [m][n] (one token)."""
    torch = _torch()
    _cuda(W, "W")
    _cuda(x, "x")
    m, n = W.shape
    if y is None:
        y = torch.empty(m, dtype=torch.float32, device=W.device)
    if xbuf is None:
        xbuf = torch.empty(n, dtype=torch.float32, device=W.device)
    _check(lib.wina_dense_matvec(_ptr(W), _dt(W), m, n, _ptr(x), _dt(x), _ptr(y), _ptr(xbuf), _stream()),
           "wina_dense_matvec")
    return y


def dense_ffn_swiglu(W_gate, W_up, W_down, x, y=None, ws: Workspace | None = None, status=None):
    """The dense comparator of the FFN on the output-major weights (one token): returns y [d]."""
    torch = _torch()
    for t_, nm in ((W_gate, "W_gate"), (W_up, "W_up"), (W_down, "W_down"), (x, "x")):
        _cuda(t_, nm)
    ffn, d = W_gate.shape
    if y is None:
        y = torch.empty(d, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = Workspace(OP_DENSE_FFN, d, ffn, 0, 1, device=x.device)
    _check(lib.wina_dense_ffn_swiglu(_ptr(W_gate), _ptr(W_up), _ptr(W_down), _dt(W_gate), d, ffn, _ptr(x), _dt(x),
                                     _ptr(y), ws.ptr, ws.nbytes, _ptr(status) if status is not None else None,
                                     _stream()), "wina_dense_ffn_swiglu")
    return y


def spark_ffn(W_gate, W_up, Wt_down, x, s: float = 0.08, ws: Workspace | None = None, status=None, y=None):
    """The Spark FFN as a key-value lookup for one token: W_gate, W_up output-major [ffn][d],
    Wt_down input-major [ffn][d]. Returns (y [d], g [ffn], idx [ffn] (first count valid),
    count [1])."""
    torch = _torch()
    for t_, nm in ((W_gate, "W_gate"), (W_up, "W_up"), (Wt_down, "Wt_down"), (x, "x")):
        _cuda(t_, nm)
    ffn, d = W_gate.shape
    if ws is None:
        ws = Workspace(OP_SPARK_FFN, d, ffn, 0, 1, device=x.device)
    if y is None:
        y = torch.empty(d, dtype=torch.float32, device=x.device)
    g = torch.empty(ffn, dtype=torch.float32, device=x.device)
    idx = torch.empty(ffn, dtype=torch.int32, device=x.device)
    count = torch.empty(1, dtype=torch.int32, device=x.device)
    _check(lib.spark_ffn_swiglu(_ptr(W_gate), _ptr(W_up), _ptr(Wt_down), _dt(W_gate), d, ffn, _ptr(x), _dt(x),
                                float(s), _ptr(y), _ptr(g), _ptr(idx), _ptr(count), ws.ptr, ws.nbytes, _ptr(status),
                                _stream()), "spark_ffn_swiglu")
    return y, g, idx, count


def ffn_ws_view(ws: Workspace, d: int, ffn: int, batch: int) -> dict:
    """Views of the intermediate results a sparse_ffn_swiglu call leaves in `ws`:
    h [B][ffn] float32; keep_gate, keep_up [B][d] and keep_down [B][ffn] as 0/1 bytes;
    the single-token kernel's phase clock stamps [16] (int64 SM cycles of CTA 0) and
    per-CTA phase end times cta_t [296][4] (int64 ns)."""
    torch = _torch()
    v = _FfnView()
    _check(lib.wina_ffn_ws_view(d, ffn, batch, ctypes.byref(v)), "wina_ffn_ws_view")
    buf = ws.buf

    def take(off, count, dtype, shape):
        nb = count * torch.empty(0, dtype=dtype).element_size()
        return buf[off: off + nb].view(dtype).view(*shape)

    return dict(
        h=take(v.h, batch * ffn, torch.float32, (batch, ffn)),
        keep_gate=take(v.keep_gate, batch * d, torch.uint8, (batch, d)),
        keep_up=take(v.keep_up, batch * d, torch.uint8, (batch, d)),
        keep_down=take(v.keep_down, batch * ffn, torch.uint8, (batch, ffn)),
        stamps=take(v.stamps, 16, torch.int64, (16,)),
        cta_t=take(v.cta_t, 296 * 4, torch.int64, (296, 4)),
    )


# ------------------------------------------------------------------------------------
# Double Sparsity decode attention
# ------------------------------------------------------------------------------------


def ds_channel_absmean(K, seq_len):
    """Mean |K| per (key/value head, channel) over the valid tokens: K [B][Hkv][Tmax][dh],
    seq_len int32 [B] -> float32 [Hkv][dh]."""
    torch = _torch()
    _cuda(K, "K")
    _cuda(seq_len, "seq_len")
    B, Hkv, Tmax, dh = K.shape
    out = torch.empty((Hkv, dh), dtype=torch.float32, device=K.device)
    _check(lib.ds_channel_absmean(_ptr(K), _dt(K), B, Hkv, Tmax, dh, _ptr(seq_len), _ptr(out), _stream()),
           "ds_channel_absmean")
    return out


def ds_calibrate_channels(K, seq_len, r: int):
    """The K-outlier channels: the r channels of largest mean |K| per key/value head,
    ascending (int32 [Hkv][r]); the means go through the top-K gate kernel."""
    a = ds_channel_absmean(K, seq_len)
    idx, _ = select_topk(a, None, r)
    return idx


def ds_label_build(K, seq_len, channels, t0: int = 0, t1: int | None = None, label=None):
    """The label cache [B][Hkv][Tmax][r] (K's dtype) for tokens [t0, t1)."""
    torch = _torch()
    for t_, nm in ((K, "K"), (seq_len, "seq_len"), (channels, "channels")):
        _cuda(t_, nm)
    B, Hkv, Tmax, dh = K.shape
    r = channels.shape[1]
    if t1 is None:
        t1 = Tmax
    if label is None:
        label = torch.zeros((B, Hkv, Tmax, r), dtype=K.dtype, device=K.device)
    _check(lib.ds_label_build(_ptr(K), _dt(K), B, Hkv, Tmax, dh, _ptr(seq_len), _ptr(channels), r, t0, t1,
                              _ptr(label), _stream()), "ds_label_build")
    return label


def ds_decode_attention(q, K, V, label, channels, seq_len, k: int, scale: float = 0.0, out=None,
                        want_idx: bool = False, want_scores: bool = False, status=None):
    """One Double Sparsity decode step: q [B][Hq][dh] -> out float32 [B][Hq][dh]; with
    want_idx / want_scores also the kept tokens [B][Hq][k] and the approximate scores
    [B][Hq][Tmax]. Returns (out, idx or None, scores or None)."""
    torch = _torch()
    for t_, nm in ((q, "q"), (K, "K"), (V, "V"), (label, "label"), (channels, "channels"), (seq_len, "seq_len")):
        _cuda(t_, nm)
    B, Hq, dh = q.shape
    _, Hkv, Tmax, _ = K.shape
    r = channels.shape[1]
    if out is None:
        out = torch.empty((B, Hq, dh), dtype=torch.float32, device=q.device)
    idx = torch.full((B, Hq, k), -1, dtype=torch.int32, device=q.device) if want_idx else None
    sc = torch.zeros((B, Hq, Tmax), dtype=torch.float32, device=q.device) if want_scores else None
    _check(lib.ds_decode_attention(_ptr(q), _dt(q), _ptr(K), _ptr(V), _ptr(label), _dt(K), _ptr(channels), B, Hq,
                                   Hkv, Tmax, dh, r, _ptr(seq_len), k, float(scale), _ptr(out),
                                   _ptr(idx) if idx is not None else None, _ptr(sc) if sc is not None else None,
                                   _ptr(status) if status is not None else None, _stream()), "ds_decode_attention")
    return out, idx, sc
