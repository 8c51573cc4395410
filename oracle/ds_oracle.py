"""Plain, slow CPU oracle (numpy) for Double Sparsity decode attention.

TEST INFRASTRUCTURE ONLY: imported solely by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference leg. The CUDA path never routes through it.
It shares no code, table or helper with the CUDA library.

Source: [DS] "大模型DoubleSparse稀疏化技术原理" (m.youleyou.com, 2026-07-13), section
技术原理: 离线校准 (offline calibration: the outlier channels of K, the label cache that
holds them contiguously) and 在线前向计算 (the decode step in three parts: the query's
important channels; approximate scores of that sparse query against the label cache;
the top-k tokens by those scores, then full attention over those tokens with the full
query, keys and values).

Readings taken where the page is silent:

* channels are chosen per key/value head by the K-outlier strategy: the r channels
  with the largest mean |K| over the calibration tokens (float64 means), ties to the
  lower channel index, listed in ascending order;
* the label cache holds the chosen channels of every token at the key cache's own
  precision (the page allows 4-bit storage but gives no quantiser);
* an approximate score is a float32 dot product computed in a fixed order: each
  product q[C_j] * label_j rounded to float32, then added to a float32 sum in channel
  order j = 0, 1, ..., r-1 (the order fixes the scores bit for bit, so that the
  top-k decision is the same on both sides);
* the top-k tokens are the k largest signed scores, ties to the lower token index,
  listed in ascending order; k >= T keeps every token;
* attention over the selected tokens is softmax(q . K_t * scale) over those tokens
  only, applied to their value rows; scale = 1 / sqrt(head dim) unless given;
* with grouped queries (several query heads per key/value head) each query head
  scores the shared label cache with its own channels' values and picks its own tokens.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "ds_channel_absmean",
    "ds_calibrate_channels",
    "ds_label_cache",
    "ds_scores",
    "ds_select_tokens",
    "ds_attention",
    "ds_decode_head",
    "ds_decode",
]


def _topk_desc_ties_low(score, k: int) -> np.ndarray:
    """Ascending indices of the k largest values (ties to the lower index)."""
    s = np.asarray(score, dtype=np.float64)
    n = s.shape[0]
    k = max(0, min(int(k), n))
    order = np.lexsort((np.arange(n), -s))  # primary key -score, secondary key index
    return np.sort(order[:k]).astype(np.int32)


# --------------------------------------------------------------------------------------
# offline calibration ([DS] 离线校准)
# --------------------------------------------------------------------------------------


def ds_channel_absmean(K) -> np.ndarray:
    """Mean |K[t, c]| over the calibration tokens t, per channel c (float64).
    K: [T][dh] values of one key/value head (any float dtype; read exactly)."""
    K64 = np.abs(np.asarray(K, dtype=np.float64))
    return K64.mean(axis=0)


def ds_calibrate_channels(K, r: int, absmean=None) -> np.ndarray:
    """The K-outlier channels of one key/value head: the r channels of largest mean |K|
    (ties to the lower channel index), ascending. ``absmean`` may be given (for
    stage-wise checks against another implementation's means)."""
    a = ds_channel_absmean(K) if absmean is None else np.asarray(absmean, dtype=np.float64)
    return _topk_desc_ties_low(a, r)


def ds_label_cache(K, channels) -> np.ndarray:
    """The label cache of one key/value head: the chosen channels of every token, stored
    contiguously ([DS]: copied from the key cache at prefill, appended at decode).
    K: [T][dh] -> [T][r], same values (a gather)."""
    return np.asarray(K)[:, np.asarray(channels, dtype=np.int64)]


# --------------------------------------------------------------------------------------
# the decode step ([DS] 在线前向计算)
# --------------------------------------------------------------------------------------


def ds_scores(q, label, channels) -> np.ndarray:
    """Step 1 and 2: the query's important channels q[C] and their approximate scores
    against every token's label row, in float32: s_t = sum over j of fl32(q[C_j] *
    label[t, j]), summed in the order j = 0..r-1 with a float32 rounding after each
    add. q: [dh] float32-exact values; label: [T][r] float32-exact values."""
    qc = np.asarray(q, dtype=np.float32)[np.asarray(channels, dtype=np.int64)]
    lab = np.asarray(label, dtype=np.float32)
    s = np.zeros(lab.shape[0], dtype=np.float32)
    for j in range(lab.shape[1]):
        s = (s + (qc[j] * lab[:, j]).astype(np.float32)).astype(np.float32)
    return s


def ds_select_tokens(scores, k: int) -> np.ndarray:
    """Step 3 (selection): the k tokens of largest approximate score (signed; ties to
    the lower token index), ascending. k >= T keeps all T tokens."""
    return _topk_desc_ties_low(np.asarray(scores, dtype=np.float32), k)


def ds_attention(q, K, V, idx, scale=None) -> np.ndarray:
    """Step 3 (attention): full-precision softmax attention of the full query over the
    selected tokens only: o = sum over t in idx of p_t V[t], p = softmax(q . K[t] * scale)
    (float64). K, V: [T][dh]."""
    q64 = np.asarray(q, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    dh = q64.shape[0]
    if idx.size == 0:
        return np.zeros(np.asarray(V).shape[1])
    sc = 1.0 / math.sqrt(dh) if scale is None else float(scale)
    K64 = np.asarray(K, dtype=np.float64)[idx]
    V64 = np.asarray(V, dtype=np.float64)[idx]
    logits = (K64 @ q64) * sc
    e = np.exp(logits - logits.max())
    p = e / e.sum()
    return p @ V64


def ds_decode_head(q, K, V, label, channels, k: int, scale=None) -> dict:
    """One query head: scores, selected tokens and the attention output."""
    s = ds_scores(q, label, channels)
    idx = ds_select_tokens(s, k)
    return dict(scores=s, idx=idx, out=ds_attention(q, K, V, idx, scale))


def ds_decode(q, K, V, label, channels, seq_len, k: int, scale=None) -> dict:
    """A decode batch: q [B][Hq][dh]; K, V [B][Hkv][Tmax][dh]; label [B][Hkv][Tmax][r];
    channels [Hkv][r]; seq_len [B] (tokens 0..seq_len[b]-1 are valid). Query head h
    reads key/value head h // (Hq / Hkv). Returns per (b, h): scores, idx, out."""
    q = np.asarray(q)
    B, Hq, dh = q.shape
    Hkv = np.asarray(K).shape[1]
    grp = Hq // Hkv
    out = np.zeros((B, Hq, dh))
    scores, idxs = {}, {}
    for b in range(B):
        T = int(seq_len[b])
        for h in range(Hq):
            g = h // grp
            r = ds_decode_head(q[b, h], K[b, g, :T], V[b, g, :T], label[b, g, :T], channels[g], k, scale)
            out[b, h] = r["out"]
            scores[(b, h)] = r["scores"]
            idxs[(b, h)] = r["idx"]
    return dict(out=out, scores=scores, idx=idxs)
