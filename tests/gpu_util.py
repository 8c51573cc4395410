"""Helpers for the GPU parity tests: uploads of the seeded inputs and error metrics.
No arithmetic of the method lives here."""

from __future__ import annotations

import numpy as np


def torch():
    import torch as _t
    return _t


def dev_bf16(bits: np.ndarray):
    """uint16 bf16 bit patterns -> a CUDA bfloat16 tensor with the same bits."""
    t = torch()
    return t.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(t.bfloat16)


def dev_f32(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_i32(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def host(t) -> np.ndarray:
    tt = torch()
    if t.dtype == tt.bfloat16:
        return t.view(tt.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    if den == 0.0:
        return float(np.linalg.norm(got))
    return float(np.linalg.norm(got - want) / den)


def status_word():
    t = torch()
    return t.zeros(1, dtype=t.int32, device="cuda")
