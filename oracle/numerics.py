"""Scalar numerics of the oracle (float64 host code).

Test infrastructure only; see ``oracle/__init__.py``.

``round_bf16`` mirrors where a bfloat16 device path stores a value: the value
is first a float32 (the device computes in float32), then rounded to bfloat16
with round-to-nearest-even.  The oracle calls it only in its ``emulate_bf16``
mode, at the storage points listed in ``oracle.model``.
"""
from __future__ import annotations

import numpy as np


def round_f32(x: np.ndarray) -> np.ndarray:
    """Round float64 values to float32 (IEEE RNE), returned as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (RNE) -> bfloat16 (RNE), returned as float64.

    bfloat16 keeps the top 16 bits of a float32.  Round-to-nearest-even on the
    dropped 16 bits: add 0x7FFF plus the lowest kept bit, then truncate.  NaN
    and infinity are passed through unchanged (the decoder never produces
    them; they are kept only so the function is total).
    """
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    finite = np.isfinite(f)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = np.where(finite, r.view(np.float32), f)
    return out.astype(np.float64)


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x)), stable for large |x|."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = x[pos] / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = x[~pos] * ex / (1.0 + ex)
    return out


def logsumexp(z: np.ndarray, axis: int = -1) -> np.ndarray:
    """log(sum(exp(z))) along ``axis`` with the usual max shift; -inf entries
    (excluded ids) contribute nothing."""
    z = np.asarray(z, dtype=np.float64)
    m = np.max(z, axis=axis, keepdims=True)
    s = np.sum(np.exp(z - m), axis=axis, keepdims=True)
    return np.squeeze(m + np.log(s), axis=axis)
