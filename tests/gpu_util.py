"""Helpers for GPU tests: build the library, create a decoder with weights."""
from __future__ import annotations

import pytest


def require_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def make_decoder(shape, weights, max_seq: int, max_batch: int = 1, env=None):
    """Decoder with weights loaded; env: variables set while the context is
    created (the library reads its kernel switches then)."""
    import os
    from kv_cache_decode_dualcache_b200 import build, fdllm
    build.build(checks=os.environ.get("FDLLM_CHECKS") == "1")
    saved = {k: os.environ.get(k) for k in (env or {})}
    os.environ.update(env or {})
    try:
        dec = fdllm.Decoder(shape, max_seq, max_batch=max_batch)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    dec.load_weights(weights)
    return dec
