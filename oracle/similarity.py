"""Similarity of K/V activations between denoising steps (oracle).

Test infrastructure only; see ``oracle/__init__.py``.

The approximate block cache rests on the observation that the K/V
activations of adjacent denoising steps are nearly the same, their cosine
similarity close to 1 (ccyt168.com Fast-dLLM overview, section 一 "核心技术",
item 1, 高相似度验证 / Fig. 2; techwalker.com Fast-dLLM article, section
"核心创新：适合扩散模型的KV缓存").  Reading taken where the pages do not say
how the cosine is formed: per layer and per position, over the vector of all
KV heads' values at that position (n_kv_heads * head_dim numbers), for K and
for V separately, each sequence's K/V coming from a full forward over it.
"""
from __future__ import annotations

from typing import List, Sequence

import numpy as np

from .model import KV, Model


def kv_cosine(kv_a: List[KV], kv_b: List[KV]) -> np.ndarray:
    """cos[layer, kv, pos] of two per-layer K/V lists ([L, Hkv, hd] arrays),
    kv = 0 for K and 1 for V; float64.  Two zero vectors count as identical
    (1), a zero and a non-zero vector as unrelated (0)."""
    if len(kv_a) != len(kv_b):
        raise ValueError("different layer counts")
    out = []
    for (ka, va), (kb, vb) in zip(kv_a, kv_b):
        per_kv = []
        for a, b in ((ka, kb), (va, vb)):
            a = np.asarray(a, dtype=np.float64).reshape(a.shape[0], -1)
            b = np.asarray(b, dtype=np.float64).reshape(b.shape[0], -1)
            dot = np.sum(a * b, axis=1)
            na = np.sqrt(np.sum(a * a, axis=1))
            nb = np.sqrt(np.sum(b * b, axis=1))
            den = na * nb
            both_zero = (na == 0) & (nb == 0)
            cos = np.where(den > 0, dot / np.where(den > 0, den, 1.0), np.where(both_zero, 1.0, 0.0))
            per_kv.append(cos)
        out.append(per_kv)
    return np.asarray(out)


def step_kv_cosine(model: Model, x_a: Sequence[int], x_b: Sequence[int]) -> np.ndarray:
    """cos[layer, kv, pos] of the K/V that full forwards over the token
    sequences x_a and x_b (same length) produce, e.g. the sequence at a block
    start (whose K/V a DualCache step reuses) and the sequence some steps
    later (the K/V a full recompute would give then)."""
    if len(x_a) != len(x_b):
        raise ValueError("sequences of different lengths")
    L = len(x_a)
    _, kv_a = model.forward(x_a, range(L), return_kv=True, head_rows=[0])
    _, kv_b = model.forward(x_b, range(L), return_kv=True, head_rows=[0])
    return kv_cosine(kv_a, kv_b)
